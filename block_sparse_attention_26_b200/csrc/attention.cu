// attention.cu -- step 3: the fine pass (exact kept blocks + centroids, one
// FP32 online softmax) and the dense rows.
//
// "minimax-h3-chunk-star7" README, section "Sol": selected K/V blocks are
// computed exactly; unselected blocks are not dropped but contribute through
// their K/V centroids, merged into the same FP32 online softmax.  Section
// "SLA": only the routed K/V blocks take part; softmax state and the final
// accumulation stay FP32.  "BlockSparseAttention - ComfyUI Built-in Node
// Documentation", general inputs, sink_conditioning: exact_kv (the packed
// prefix blocks arrive here as kept blocks) and exact_kv_and_rows (designated
// query rows run dense and replace the sparse result).
//
// Work items (one CTA each, one CTA per SM):
//   dense item   128 rows of the dense range x one chunk of the key blocks;
//                with more than one chunk it writes an unnormalised partial
//                (O, m, l) that combine_kernel merges, so that the few dense
//                rows spread over the whole GPU;
//   sparse item  128 query rows of one (batch, head): two 64-row query blocks
//                (Sol, Q64) or one 128-row block (SLA, Q128), so that every
//                tensor-core instruction has M = 128.  It walks the sorted union
//                of its query blocks' kept key blocks, then the centroid chunks.
// Dense items come first in the grid so that they start early.
//
// A tile is 128 keys: two key blocks (or two chunks of 64 centroids) loaded
// into the two halves of the K and V tiles, so that S = Q K^T is an N = 128
// UMMA (N = 64 UMMAs run at two thirds of the rate).  Softmax warpgroup h owns
// the tile's half h -- one key block -- with its own online softmax state and
// its own accumulator O_h; the halves are merged in the epilogue.
//
// Warp roles (352 threads):
//   warps 0-3, 4-7  softmax warpgroups h = 0, 1: thread r owns query row r
//              (TMEM lane r).  Read S from TMEM, mask, online softmax in the log2
//              domain with a lazily updated reference max (the accumulator is
//              rescaled only when the row max grows by more than 2^8), write P
//              (bf16) into TMEM, and run the epilogue.
//   warps 8, 10  K and V producers: each builds the same tile list and TMA-loads
//              its K (resp. V) tiles (or bf16 centroid tiles) into its own ring,
//              so K prefetch never waits for V slots; a K slot is released as
//              soon as its S product is done, the V producer also publishes each
//              tile's masks to the softmax warps.
//   warp 9     MMA issuer (fixed order; the whole warp runs it, one elected
//              lane issues): S = Q K^T (A and B from
//              shared memory) runs one tile ahead of the softmax, into two TMEM
//              buffers; per tile j it issues O_h += P_h V_h (A = P_h from TMEM)
//              for h = 0, 1, then S(j + 2) into the buffer P(j) held: the tensor
//              pipe runs one thread's MMAs in issue order.  All of that waits on one
//              barrier, ready(j): both halves' P(j) written and K(j + 2) landed (or
//              the list's end reached).  The tensor pipe takes only a couple of
//              MMAs ahead of its issuer, so every wait between MMA groups leaves it
//              idle for about a barrier round trip: one wait per tile, not three.
//              The completion of S(j) also frees K slot j % 2, and the
//              completion of S(j + 1) tells a softmax warp that wants to rescale
//              O at tile j that P V(j - 1) is done.
// TMEM (512 columns): S of tile j at 128 (j & 1), half h's P (bf16 pairs) written
// over its own S columns 128 (j & 1) + 64 h once read; O_h at 256 + 128 h.
#include <math.h>

#include <algorithm>

#include <cuda_fp8.h>

#include "bsa_device.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kM = 128;        // query rows per tile (UMMA M)
constexpr int kBK = 64;        // keys per key block
constexpr int kTK = 128;       // keys per tile (two blocks)
constexpr int kKS = 2;         // K ring depth (tiles)
constexpr int kVS = 3;         // V ring depth (tiles)
constexpr int kThreads = 352;  // 2 softmax warpgroups + K producer + MMA + V producer
constexpr float kRescaleLog2 = 8.0f;
constexpr float kOptSum = 16777216.0f;   // 2^24: bound on a bf16 tile's sum of P without its maximum
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;          // S of tile j at kColS + 128 (j & 1); P of half h over its own S
constexpr uint32_t kColO = 256;        // O of half h at kColO + 128 h

enum : int32_t { TILE_EXACT = 0, TILE_CENT = 1, TILE_END = 2, TILE_GATHER = 3 };
constexpr int kMaxE = 256;     // extra tokens per query block (the node's range is 0..256)

#ifdef BSA_TRACE
// Per-tile clock64() stamps of a few CTAs (development builds only), kept in
// shared memory while the CTA runs and copied out at its end.
#ifndef BSA_TRACE_TILES
#define BSA_TRACE_TILES 64
#endif
constexpr int kTraceCtas = 8, kTraceTiles = BSA_TRACE_TILES, kTraceEvents = 16;
constexpr int kTraceBytes = kTraceTiles * kTraceEvents * 8;
#define TRACE(ev, j)                                                                       \
    do {                                                                                   \
        if ((j) < kTraceTiles) trace_sm[(ev) * kTraceTiles + (j)] = clock64();              \
    } while (0)
#else
constexpr int kTraceBytes = 0;
#define TRACE(ev, j) ((void)0)
#endif

// What one 128-key tile holds; half h is one key block (or 64 centroids).
struct TileInfo {
    // per half, read by its softmax warps with one 16-byte load: {kind, who (exact:
    // bit q set = query block q of the tile keeps the half's block), ncols (exact:
    // valid key columns, 0 = empty half), pcol (centroid: column of a partial block,
    // or -1)}
    int4 h[2];
    int32_t blk[2];       // key block of each half (exact) or centroid chunk (centroid)
    float last_bias;      // centroid: log2 of the partial block's size
    int32_t pad;
    uint64_t cmask[2][2]; // centroid / gathered: [query block][half] active columns
    float ksc[2];         // fp8 Q K^T: scale of each half's keys (1 otherwise)
    int32_t pad2[2];
};

struct AttnArgs {
    int B, H, N, nQB, nKB, nW, Bq;
    int64_t sb, sn, sh;          // output element strides
    const int64_t *row_ptr;
    const int32_t *col_idx;
    void *out;
    float *lse;
    int out_f32;
    int centroid;
    int n_sparse;                // sparse items per (b, h)
    int skip_begin, skip_end;    // sparse tiles fully inside are left to the dense items
    int dense_begin, dense_end;  // dense rows
    int n_dense;                 // dense row tiles per (b, h)
    int dense_split;             // key chunks per dense row tile
    int split_blocks;            // key blocks per chunk
    float *part_o;               // [tiles, split, 128, d] unnormalised partial outputs
    float *part_ml;              // [tiles, split, 128, 2] (m, l) in the log2 domain
    float scale_log2;            // log2(e) / sqrt(d)
    int32_t *status;
    long long *trace;            // development builds: per-tile timestamps
    int trace_base;
    // extra tokens (E > 0): gathered as exact keys; the blocks they came from keep a
    // centroid over their remaining tokens (per query block)
    int E, Ecap;
    const int32_t *extra_idx;    // [rows, E] ascending token indices
    const int32_t *extra_count;  // [rows]
    const __nv_bfloat16 *kx, *vx;              // K and V inputs (bf16), output strides
    const __nv_bfloat16 *xk16, *xv16;          // [mc_cap, d] modified centroids
    const float *xbias;                        // [mc_cap] log2 of their token counts
    const int32_t *xcnt;                       // [rows] modified centroids per row
    const int64_t *xoff;                       // [rows] where row r's start
    const int32_t *slot;                       // [mc_cap] their places in xk16 / xv16
    // gathers by TMA (tile::gather4) when K and V are one uniform 2-D array of token
    // rows: row of (b, n, h) = b grow_b + n grow_n + h grow_h; else by cp.async
    int gather_tma;
    int64_t grow_b, grow_n, grow_h;
    const uint32_t *glist;                     // [sparse tiles, kGlistCap] extra-token union per tile
    const int32_t *glcnt;                      // [sparse tiles] its length (a multiple of 4)
    // cube tiling (vsa): positions are in block order (the prefix's 64-token
    // blocks, then the grid's cubes); tiles of cubes come through 5-D maps
    int cube, pre_blocks, P, gH, gW, cT, cH, cW, ncx, ncy;
    // fp8 Q K^T: scales of Q per 64 tokens, of K per key block, of the centroids per 64
    const float *sq8, *sk8, *skc8;
    int nb64, nch64;
    // fp8 P V: scale of V per (b, h, channel)
    const float *sv8;
};

// Token of block-order position p (identity without cube tiling).
__device__ __forceinline__ int pos_token(const AttnArgs &a, int p)
{
    if (!a.cube) return p;
    const int blk = p >> 6, t = p & 63;
    if (blk < a.pre_blocks) return p;
    const int c = blk - a.pre_blocks;
    const int cx = c % a.ncx, cy = (c / a.ncx) % a.ncy, ct = c / (a.ncx * a.ncy);
    const int dx = t % a.cW, dy = (t / a.cW) % a.cH, dt = t / (a.cW * a.cH);
    return a.P + ((ct * a.cT + dt) * a.gH + cy * a.cH + dy) * a.gW + cx * a.cW + dx;
}

// 64 rows from block-order position pos through the 4-D map (64-row box) when
// they are prefix tokens (any pos) or past the end (zeros), else the cube that
// starts at pos (a multiple of 64) through the 5-D map.
__device__ __forceinline__ void load_rows64(uint8_t *dst, const AttnArgs &a, const CUtensorMap *m4,
                                            const CUtensorMap *m5, uint64_t *bar, int dc, int h, int b, int pos)
{
    if (pos < a.P || pos >= a.N) {
        tma_load_4d(dst, m4, bar, dc * 64, h, pos, b);
    } else {
        const int c = (pos >> 6) - a.pre_blocks;
        const int cx = c % a.ncx, cy = (c / a.ncx) % a.ncy, ct = c / (a.ncx * a.ncy);
        tma_load_5d(dst, m5, bar, dc * 64, h, cx * a.cW, cy * a.cH, ct * a.cT);
    }
}

template <int D, bool QK8 = false, bool PV8 = false>
struct Lay {
    // Q and K tiles hold 1 byte per channel with fp8 Q K^T (QK8), else 2; V tiles
    // 1 byte with fp8 P V (PV8)
    static constexpr int kQKElem = QK8 ? 1 : 2;
    static constexpr int kQBytes = kM * D * kQKElem;
    static constexpr int kKTileBytes = kTK * D * kQKElem;       // one K tile (128 keys)
    static constexpr int kTileBytes = kTK * D * (PV8 ? 1 : 2);  // one V tile (128 keys)
    static constexpr int kHalfBytes = kBK * 128;                // one 64-key box of one 128-byte channel chunk
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kKS * kKTileBytes;
    static constexpr int kOffKind = kOffV + kVS * kTileBytes;
    static constexpr int kOffInfo = kOffKind + 16;
    static constexpr int kOffBar = kOffInfo + kVS * (int)sizeof(TileInfo);
    // q, done, k_full[KS], v_full[VS], v_empty[VS], s_full[2 buffers], ready[2 buffers]
    static constexpr int kNumBar = 2 + kKS + 2 * kVS + 2 + 2;
    static constexpr int kOffMisc = kOffBar + kNumBar * 8;
    static constexpr int kOffML = kOffMisc + 16;                 // [2][128] (m, l) per half
    static constexpr int kOffBias = kOffML + 2 * kM * 8;         // [VS][128] per-column bias (gathers)
    // gathered columns of the CTA: the union of its query blocks' extra tokens, then
    // each query block's modified centroids (code, query-block bits, bias source)
    static constexpr int kOffGlCode = kOffBias + kVS * kTK * 4;   // [4 kMaxE] u32
    static constexpr int kOffGlBias = kOffGlCode + 4 * kMaxE * 4; // [2][kMaxE] modified-centroid biases
    static constexpr int kOffGlWho = kOffGlBias + 2 * kMaxE * 4;  // [4 kMaxE] u8
    static constexpr int kOffExt = kOffGlWho + 4 * kMaxE;         // [8] list lengths
    static constexpr int kOffTrace = kOffExt + 32;
    static constexpr int kOffMask = kOffTrace + kTraceBytes;     // kept [2][nW], then affected [2][nW]
    // at least 116 KB so that a single CTA owns an SM (it allocates all 512 TMEM columns)
    static size_t bytes(int nW)
    {
        const size_t b = (size_t)kOffMask + 4 * (size_t)nW * 4 + 1024;
        return b < 116 * 1024 ? 116 * 1024 : b;
    }
};

// 2^x on the MUFU unit (ex2.approx, relative error ~2^-22; 2^-inf = +0).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Non-blocking test of two barrier phases and a 16-byte shared-memory load in
// one sequence; true if both phases are complete, and only then is the value
// meaningful (the load is ordered after the tests' acquire).  The three accesses
// overlap instead of taking a round trip each.
__device__ __forceinline__ bool test2_load16(uint64_t *b0, uint32_t p0, uint64_t *b1, uint32_t p1, const void *src,
                                             int4 &v)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred a, b;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 a, [%5], %6;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 b, [%7], %8;\n\t"
        "ld.volatile.shared.v4.s32 {%0, %1, %2, %3}, [%9];\n\t"
        "and.pred a, a, b;\n\t"
        "selp.u32 %4, 1, 0, a;\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w), "=r"(ok)
        : "r"(smem_u32(b0)), "r"(p0), "r"(smem_u32(b1)), "r"(p1), "r"(smem_u32(src))
        : "memory");
    return ok != 0;
}

// UMMA issue in warp-wide form: every lane of the warp executes these with the
// same operands and one elected lane issues (the operands stay warp-uniform).
// D[tmem] (+)= A[smem] * B[smem]^T.
__device__ __forceinline__ void umma_ss_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// The same with fp8 (e4m3) operands, K = 32 per instruction.
__device__ __forceinline__ void umma_ss_f8_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Instruction descriptor, kind::f8f6f4 with e4m3 A and B (K-major) and f32 accumulate.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N)
{
    return (1u << 4)                       // D format f32
           | (0u << 7)                     // A format e4m3
           | (0u << 10)                    // B format e4m3
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M x K, bf16 pairs per 32-bit column) from TMEM.
__device__ __forceinline__ void umma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// The same with e4m3 operands (kind::f8f6f4, K = 32): A (4 values a 32-bit column) from TMEM.
__device__ __forceinline__ void umma_ts_f8_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` once every tcgen05 operation the warp issued so far completes.
__device__ __forceinline__ void umma_commit_w(uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

// Packed pairs of f32 (one instruction for two values; round to nearest).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float fmax3(float x, float y, float z)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(x), "f"(y), "f"(z));
    return r;
}

// Maximum of 64 values with three-input max instructions (32 of them).
__device__ __forceinline__ float max64(const float (&x)[64])
{
    float m[22];
#pragma unroll
    for (int i = 0; i < 21; ++i) m[i] = fmax3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
    m[21] = x[63];
    float n[8];
#pragma unroll
    for (int i = 0; i < 7; ++i) n[i] = fmax3(m[3 * i], m[3 * i + 1], m[3 * i + 2]);
    n[7] = m[21];
    const float a = fmax3(n[0], n[1], n[2]), b = fmax3(n[3], n[4], n[5]);
    return fmax3(a, b, fmaxf(n[6], n[7]));
}

__device__ __forceinline__ void named_bar(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int D, bool QK8, bool PV8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_gk,
                const __grid_constant__ CUtensorMap tm_gv, const __grid_constant__ CUtensorMap tm_gxk,
                const __grid_constant__ CUtensorMap tm_gxv, const __grid_constant__ CUtensorMap tm_q5,
                const __grid_constant__ CUtensorMap tm_k5, const __grid_constant__ CUtensorMap tm_v5,
                const AttnArgs a)
{
    using L = Lay<D, QK8, PV8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ------------------------------------------------------------ work item
    int64_t item = blockIdx.x;
    const int64_t nd_items = (int64_t)a.B * a.H * a.n_dense * a.dense_split;
    const bool dense = item < nd_items;
    int bh, row0, nvalid, kb0 = 0, kb1 = 0;
    int64_t pidx = 0, sidx = 0;   // dense partial index; sparse tile index (b, h, tile)
    if (dense) {
        const int split = (int)(item % a.dense_split);
        const int64_t tt = item / a.dense_split;          // (bh, tile)
        const int t = (int)(tt % a.n_dense);
        bh = (int)(tt / a.n_dense);
        row0 = a.dense_begin + t * kM;
        nvalid = min(kM, a.dense_end - row0);
        kb0 = split * a.split_blocks;
        kb1 = min(a.nKB, kb0 + a.split_blocks);
        pidx = tt * a.dense_split + split;
    } else {
        item -= nd_items;
        sidx = item;
        const int tile = (int)(item % a.n_sparse);
        bh = (int)(item / a.n_sparse);
        row0 = tile * kM;
        if (row0 >= a.skip_begin && min(row0 + kM, a.N) <= a.skip_end) return;   // all rows dense
        nvalid = min(kM, a.N - row0);
    }
    const int b = bh / a.H, h = bh % a.H;
    const int qb0 = row0 / a.Bq;
    const int nq = dense ? 1 : ((a.Bq == 64 && qb0 + 1 < a.nQB) ? 2 : 1);
    const int64_t rbase = (int64_t)bh * a.nQB + qb0;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kOffBar);
    uint64_t *bar_q = bars, *bar_done = bars + 1;
    uint64_t *k_full = bars + 2;
    uint64_t *v_full = k_full + kKS, *v_empty = v_full + kVS;
    uint64_t *s_full = v_empty + kVS;         // [buffer]
    // [buffer] tile j's phase of ready[j & 1]: P(j) from all 8 softmax warps, and the
    // K producer's tile j + 2 (its TMA bytes, or an arrival past the list's end);
    // tiles 0 and 1 land on k_full
    uint64_t *ready = s_full + 2;
    volatile int32_t *kkind = reinterpret_cast<volatile int32_t *>(sm + L::kOffKind);
    volatile TileInfo *info = reinterpret_cast<volatile TileInfo *>(sm + L::kOffInfo);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kOffMisc);
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(sm + L::kOffMisc + 4);
    float2 *ml = reinterpret_cast<float2 *>(sm + L::kOffML);   // [2 halves][128] (m, l)
    uint32_t *kept = reinterpret_cast<uint32_t *>(sm + L::kOffMask);
    uint32_t *aff = kept + 2 * a.nW;                            // blocks that gave extra tokens
    float *bias_sm = reinterpret_cast<float *>(sm + L::kOffBias);
    // [0..1] extra tokens, [2..3] modified centroids per query block; [4] union size
    // (padded), [5] gathered columns in all
    int32_t *ext_n = reinterpret_cast<int32_t *>(sm + L::kOffExt);
    uint32_t *gl_code = reinterpret_cast<uint32_t *>(sm + L::kOffGlCode);
    float *gl_bias = reinterpret_cast<float *>(sm + L::kOffGlBias);
    uint8_t *gl_who = sm + L::kOffGlWho;
#ifdef BSA_TRACE
    long long *trace_sm = reinterpret_cast<long long *>(sm + L::kOffTrace);
    for (int i = threadIdx.x; i < kTraceTiles * kTraceEvents; i += blockDim.x) trace_sm[i] = 0;
#endif

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_done, 1);
        for (int s = 0; s < kKS; ++s) mbar_init(&k_full[s], 1);
        for (int s = 0; s < kVS; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&ready[0], 9);
        mbar_init(&ready[1], 9);
        *abort_flag = 0;
        fence_mbar_init();
        // Q first: its load overlaps the rest of the set-up
        prefetch_tmap(&tm_q);
        mbar_expect_tx(bar_q, L::kQBytes);
        if (QK8) {
            // 128 rows of 128 fp8 channels: one box
            tma_load_4d(sm + L::kOffQ, &tm_q, bar_q, 0, h, row0, b);
        } else if (a.cube) {
            // two 64-row blocks (the map's box is 64 rows in this mode)
            for (int dc = 0; dc < D / 64; ++dc)
                for (int half = 0; half < 2; ++half)
                    load_rows64(sm + L::kOffQ + dc * (kM * 128) + half * (64 * 128), a, &tm_q, &tm_q5, bar_q, dc, h,
                                b, row0 + 64 * half);
        } else {
            for (int dc = 0; dc < D / 64; ++dc)
                tma_load_4d(sm + L::kOffQ + dc * (kM * 128), &tm_q, bar_q, dc * 64, h, row0, b);
        }
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && !dense) {
        // kept-block bitmasks of the tile's query blocks, from the CSR lists; with
        // extra tokens also their lists and the blocks they came from.  Two rounds
        // of loads: the CSR ranges and list lengths, then every list at once.
        for (int w = lane; w < 4 * a.nW; w += 32) kept[w] = 0u;
        if (lane < 8) ext_n[lane] = 0;
        int64_t pr = 0;
        int len = 0;
        if (lane <= nq) pr = a.row_ptr[rbase + lane];
        if (a.E > 0) {
            if (lane >= 8 && lane < 8 + nq) len = a.xcnt[rbase + lane - 8];
            else if (lane >= 10 && lane < 10 + nq) len = a.extra_count[rbase + lane - 10];
            else if (lane == 12) len = a.glcnt[sidx];
        }
        const int64_t p0 = __shfl_sync(0xffffffffu, pr, 0), p2 = __shfl_sync(0xffffffffu, pr, nq);
        const int64_t p1 = nq > 1 ? __shfl_sync(0xffffffffu, pr, 1) : p2;   // query block 1's list starts there
        const int nx0 = min(__shfl_sync(0xffffffffu, len, 8), a.Ecap);
        const int nx1 = nq > 1 ? min(__shfl_sync(0xffffffffu, len, 9), a.Ecap) : 0;
        const int ec0 = min(__shfl_sync(0xffffffffu, len, 10), a.E);
        const int ec1 = nq > 1 ? min(__shfl_sync(0xffffffffu, len, 11), a.E) : 0;
        const int U = __shfl_sync(0xffffffffu, len, 12);
        int64_t xo = 0;
        if (a.E > 0 && lane >= 13 && lane < 13 + nq) xo = a.xoff[rbase + lane - 13];
        const int64_t xo0 = __shfl_sync(0xffffffffu, xo, 13), xo1 = __shfl_sync(0xffffffffu, xo, 14);
        __syncwarp();
        // the column lists of both query blocks (contiguous in the CSR), 16 in flight per lane
        for (int64_t pb = p0; pb < p2; pb += 512) {
            int cv[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int64_t p = pb + 32 * u + lane;
                cv[u] = p < p2 ? a.col_idx[p] : -2;
            }
            // the extra-token lists ride along with the first batch
            float xb[16];
            uint32_t gv[17];
            if (a.E > 0 && pb == p0) {
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int e = 32 * (u & 7) + lane;
                    const int q = u >> 3;
                    xb[u] = e < (q ? nx1 : nx0) ? a.xbias[(q ? xo1 : xo0) + e] : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 17; ++u) {
                    const int i = 32 * u + lane;
                    gv[u] = i < U ? a.glist[sidx * kGlistCap + i] : 0u;
                }
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int c = cv[u];
                if (c == -2) continue;   // past the lists
                const int q = pb + 32 * u + lane < p1 ? 0 : 1;
                if (c >= 0 && c < a.nKB)
                    atomicOr(&kept[q * a.nW + (c >> 5)], 1u << (c & 31));
                else
                    report(a.status, BSA_DEV_INTERNAL, 1);
            }
            if (a.E > 0 && pb == p0) {
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int e = 32 * (u & 7) + lane;
                    const int q = u >> 3;
                    if (e < (q ? nx1 : nx0)) gl_bias[q * kMaxE + e] = xb[u];
                }
#pragma unroll
                for (int u = 0; u < 17; ++u) {
                    const int i = 32 * u + lane;
                    if (i < U) {
                        gl_code[i] = gv[u] & 0x3fffffffu;
                        gl_who[i] = (uint8_t)(gv[u] >> 30);
                    }
                }
            }
        }
        if (a.E > 0) {
            if (p0 >= p2) {   // no kept block at all: the lists did not ride along
                for (int q = 0; q < nq; ++q)
                    for (int e = lane; e < (q ? nx1 : nx0); e += 32)
                        gl_bias[q * kMaxE + e] = a.xbias[(q ? xo1 : xo0) + e];
                for (int i = lane; i < U; i += 32) {
                    const uint32_t v = a.glist[sidx * kGlistCap + i];
                    gl_code[i] = v & 0x3fffffffu;
                    gl_who[i] = (uint8_t)(v >> 30);
                }
            }
            // blocks that gave extra tokens, per query block, from the union list
            __syncwarp();
            for (int i = lane; i < U; i += 32) {
                const uint32_t who = gl_who[i];
                const int kb = (int)(gl_code[i] >> 6);
                if (who & 1u) atomicOr(&aff[kb >> 5], 1u << (kb & 31));
                if (who & 2u) atomicOr(&aff[a.nW + (kb >> 5)], 1u << (kb & 31));
            }
            // gathered columns: the union of the query blocks' extra tokens (merged
            // by glist_kernel, padded to a multiple of 4), then each query block's
            // modified centroids
            const int m0 = nx0, m1 = nx1;
            for (int e = lane; e < m0; e += 32) {
                gl_code[U + e] = 0x80000000u | (uint32_t)a.slot[xo0 + e];
                gl_who[U + e] = 1;
            }
            for (int e = lane; e < m1; e += 32) {
                gl_code[U + m0 + e] = 0xC0000000u | (uint32_t)a.slot[xo1 + e];
                gl_who[U + m0 + e] = 2;
            }
            if (lane == 0) {
                ext_n[0] = ec0;
                ext_n[1] = ec1;
                ext_n[2] = nx0;
                ext_n[3] = nx1;
                ext_n[4] = U;
                ext_n[5] = U + m0 + m1;
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8 || warp == 10) {
        // ---------------------------------------------------------- producers
        // Every lane walks the same tile list; lane 0 waits on the ring, issues the
        // TMA loads and publishes tile metadata; all lanes copy gathered rows.
        const bool is_k = warp == 8;
        if (lane == 0) {
            if (is_k) {
                prefetch_tmap(&tm_k);
                if (!dense && a.centroid) prefetch_tmap(&tm_kc);
            } else {
                prefetch_tmap(&tm_v);
                if (!dense && a.centroid) prefetch_tmap(&tm_vc);
            }
        }
        const CUtensorMap *tm_x = is_k ? &tm_k : &tm_v;
        const CUtensorMap *tm_c = is_k ? &tm_kc : &tm_vc;
        const CUtensorMap *tm_gx = is_k ? &tm_gk : &tm_gv;     // token rows, for gathers
        const CUtensorMap *tm_gc = is_k ? &tm_gxk : &tm_gxv;   // modified-centroid rows
        const int depth = is_k ? kKS : kVS;
        uint64_t *full = is_k ? k_full : v_full;
        // a K slot is free once the S product that read it is done (S(j) sits in
        // buffer j & 1 = slot j % 2)
        static_assert(kKS == 2, "K slots and S buffers must pair up");
        uint64_t *empty = is_k ? s_full : v_empty;
        uint8_t *ring = sm + (is_k ? L::kOffK : L::kOffV);
        int gl0 = 0, gln = 0, glU = 0, glm0 = 0;   // the gathered tile: list entries [gl0, gl0 + gln)
        const __nv_bfloat16 *src_x = is_k ? a.kx : a.vx;
        const __nv_bfloat16 *src_c = is_k ? a.xk16 : a.xv16;
        int j = 0;
        // half x of the tile lands at row offset 64 x of every channel chunk
        const CUtensorMap *tm_x5 = is_k ? &tm_k5 : &tm_v5;
        auto load_half = [&](uint8_t *dst, int kind, int blk, uint64_t *bar) {
            if ((QK8 && is_k) || (PV8 && !is_k)) {
                // 64 keys of 128 fp8 channels: one box
                if (kind == TILE_EXACT)
                    tma_load_4d(dst, tm_x, bar, 0, h, blk * kBK, b);
                else
                    tma_load_3d(dst, tm_c, bar, 0, blk * kBK, bh);
                return;
            }
            for (int dc = 0; dc < D / 64; ++dc) {
                uint8_t *d = dst + dc * (kTK * 128);
                if (kind == TILE_EXACT) {
                    if (a.cube)
                        load_rows64(d, a, tm_x, tm_x5, bar, dc, h, b, blk * kBK);
                    else
                        tma_load_4d(d, tm_x, bar, dc * 64, h, blk * kBK, b);
                } else {
                    tma_load_3d(d, tm_c, bar, dc * 64, blk * kBK, bh);
                }
            }
        };
        // row address of a gathered column: an extra token of this head, or a
        // modified centroid (bit 31 set; query block in bit 30, its slot in bits 0-29)
        auto row_src = [&](uint32_t code) -> const __nv_bfloat16 * {
            if (code & 0x80000000u) return src_c + (int64_t)(code & 0x3fffffffu) * D;
            return src_x + (int64_t)b * a.sb + (int64_t)code * a.sn + (int64_t)h * a.sh;
        };
        auto push = [&](int kind, const int (&blk)[2], const uint32_t (&who)[2], const int (&nc)[2],
                        const int (&pcol)[2], float last_bias, const uint64_t (&cm)[2][2]) -> bool {
            const int s = j % depth;
            if (j >= depth) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&empty[s], ((j / depth) - 1) & 1, abort_flag, a.status, is_k ? 10 : 11);
                if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
            }
            if (lane == 0) {
                if (is_k) {
                    kkind[s] = kind;
                    TRACE(0, j);
                } else {
                    TRACE(1, j);
                    for (int x = 0; x < 2; ++x) {
                        float ksc = 1.f;
                        if (QK8 && blk[x] >= 0)
                            ksc = kind == TILE_EXACT ? a.sk8[(int64_t)bh * a.nKB + blk[x]]
                                                     : a.skc8[(int64_t)bh * a.nch64 + blk[x]];
                        info[s].ksc[x] = ksc;
                        info[s].blk[x] = blk[x];
                        info[s].h[x].x = kind;
                        info[s].h[x].y = (int32_t)who[x];
                        info[s].h[x].z = nc[x];
                        info[s].h[x].w = pcol[x];
                        info[s].cmask[x][0] = cm[x][0];
                        info[s].cmask[x][1] = cm[x][1];
                    }
                    info[s].last_bias = last_bias;
                }
            }
            uint8_t *dst = ring + s * (is_k ? L::kKTileBytes : L::kTileBytes);
            // K tile j >= 2 completes tile j - 2's ready barrier (the slot wait above
            // ordered it after that barrier's previous phase: S(j - 2) was issued after it)
            uint64_t *fb = (is_k && j >= 2) ? &ready[j & 1] : &full[s];
            if (kind == TILE_GATHER && !is_k)
                for (int c = lane; c < kTK; c += 32) {
                    // bias 0 for extra tokens, log2 of the remaining count for modified centroids
                    const int g = gl0 + c;
                    float bs = 0.f;
                    if (c < gln && g >= glU) bs = g < glU + glm0 ? gl_bias[g - glU] : gl_bias[kMaxE + g - glU - glm0];
                    bias_sm[s * kTK + c] = bs;
                }
            if (kind == TILE_GATHER && a.gather_tma) {
                // 128 rows by TMA, 4 rows per gather: lane l takes columns 4l..4l+3
                // (unused columns repeat the last entry; the 4 rows of a gather come
                // from one array because the column list is 4-aligned per array)
                if (lane == 0) mbar_expect_tx(fb, L::kTileBytes);
                __syncwarp();
                const int c = 4 * lane;
                int rw[4];
                bool cent = false;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t code = gl_code[c + i < gln ? gl0 + c + i : gl0 + gln - 1];
                    if (i == 0) cent = (code & 0x80000000u) != 0u;
                    rw[i] = cent ? (int)(code & 0x3fffffffu)
                                 : (int)(b * a.grow_b + h * a.grow_h + (int64_t)code * a.grow_n);
                }
#pragma unroll
                for (int dc = 0; dc < D / 64; ++dc)
                    tma_gather4(dst + dc * (kTK * 128) + c * 128, cent ? tm_gc : tm_gx, fb, dc * 64, rw);
            } else if (kind == TILE_GATHER) {
                // 128 rows from arbitrary addresses, written in the 128-byte-swizzled
                // layout the tensor core reads; completion through the barrier.  Unused
                // columns repeat the first row (a valid address; no column active).
                // lane l copies 16-byte chunk l % (D/8) of rows l / (D/8) + (32/(D/8)) i: the
                // row codes and addresses of a batch are formed before its copies issue
                const uint32_t base = smem_u32(dst);
                constexpr int kCh = D / 8, kRowsPerPass = 32 / kCh, kBatch = 16;
                const int k16 = lane % kCh, dc = k16 >> 3, c16 = k16 & 7;
                const uint32_t sbase = base + dc * (kTK * 128);
#pragma unroll 1
                for (int c0 = lane / kCh; c0 < kTK; c0 += kRowsPerPass * kBatch) {
                    const __nv_bfloat16 *ga[kBatch];
#pragma unroll
                    for (int i = 0; i < kBatch; ++i) {
                        const int c = c0 + kRowsPerPass * i;
                        ga[i] = row_src(gl_code[c < gln ? gl0 + c : gl0]) + k16 * 8;
                    }
#pragma unroll
                    for (int i = 0; i < kBatch; ++i) {
                        const int c = c0 + kRowsPerPass * i;
                        const uint32_t sa = sbase + (c >> 3) * 1024 + (c & 7) * 128 + ((c16 ^ (c & 7)) << 4);
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(ga[i]));
                    }
                }
                // each lane's copies complete the slot asynchronously (one pending
                // arrival per lane, added now); lane 0 gives the barrier's own arrival.
                // The MMA warp orders them before its tensor-core reads with a proxy fence.
                asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(fb)) : "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(fb);
            } else if (lane == 0) {
                if (kind == TILE_END) {
                    mbar_arrive(fb);
                } else {
                    mbar_expect_tx(fb, is_k ? L::kKTileBytes : L::kTileBytes);
                    load_half(dst, kind, blk[0], fb);
                    load_half(dst + L::kHalfBytes, kind, blk[1], fb);
                }
            }
            ++j;
            return true;
        };
        const uint64_t zero2[2][2] = {{0, 0}, {0, 0}};
        const int none[2] = {-1, -1};
        bool ok = true;
        // Gathered tiles (128 entries of the CTA's column list each) are spread
        // evenly among the exact tiles, so that each has the tiles before it to
        // arrive from DRAM.
        int gat_est = 0, gdone = 0, G = -1, n_exact = 0, exact_pushed = 0;
        if (!dense && a.E > 0) {
            gat_est = (ext_n[5] + kTK - 1) / kTK;
            int nb = 0;
            for (int w = lane; w < a.nW; w += 32) nb += __popc(kept[w] | kept[a.nW + w]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) nb += __shfl_xor_sync(0xffffffffu, nb, o);
            n_exact = (nb + 1) / 2;
        }
        auto push_gather = [&]() -> bool {
            if (G < 0) {
                G = ext_n[5];
                glU = ext_n[4];
                glm0 = ext_n[2];
            }
            const int g0 = gdone * kTK;
            if (g0 >= G) {   // fewer than the bound
                gdone = gat_est;
                return true;
            }
            gl0 = g0;
            gln = min(kTK, G - g0);
            uint64_t cm[2][2];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c = 32 * k + lane;
                const uint32_t who = c < gln ? gl_who[g0 + c] : 0u;
                const uint64_t w1 = __ballot_sync(0xffffffffu, who & 1u), w2 = __ballot_sync(0xffffffffu, who & 2u);
                if (k & 1) {
                    cm[0][k >> 1] |= w1 << 32;
                    cm[1][k >> 1] |= w2 << 32;
                } else {
                    cm[0][k >> 1] = w1;
                    cm[1][k >> 1] = w2;
                }
            }
            const int none2[2] = {-1, -1};
            const int nc0[2] = {0, 0};
            const uint32_t wh0[2] = {0u, 0u};
            ++gdone;
            return push(TILE_GATHER, none2, wh0, nc0, none2, 0.f, cm);
        };
        auto after_exact = [&]() {
            ++exact_pushed;
            while (ok && gdone < gat_est && exact_pushed >= ((gdone + 1) * n_exact) / (gat_est + 1))
                ok = push_gather();
        };
        // exact tiles: pairs of key blocks; an odd last tile repeats its block
        // in the empty half (a valid load) with no active column
        int pend = -1;
        uint32_t pend_who = 0;
        auto emit_block = [&](int blk, uint32_t who) {
            if (pend < 0) {
                pend = blk;
                pend_who = who;
                return;
            }
            const int bl[2] = {pend, blk};
            const uint32_t wh[2] = {pend_who, who};
            const int nc[2] = {min(kBK, a.N - pend * kBK), min(kBK, a.N - blk * kBK)};
            ok = push(TILE_EXACT, bl, wh, nc, none, 0.f, zero2);
            pend = -1;
            if (ok) after_exact();
        };
        if (dense) {
            for (int blk = kb0; blk < kb1 && ok; ++blk) emit_block(blk, 3u);
        } else {
            const uint32_t *k0 = kept, *k1 = kept + a.nW;
            for (int w = 0; w < a.nW && ok; ++w) {
                uint32_t u = k0[w] | k1[w];
                while (u && ok) {
                    const int bit = __ffs(u) - 1;
                    u &= u - 1;
                    emit_block(w * 32 + bit, ((k0[w] >> bit) & 1u) | (((k1[w] >> bit) & 1u) << 1));
                }
            }
        }
        if (ok && pend >= 0) {
            const int bl[2] = {pend, pend};
            const uint32_t wh[2] = {pend_who, 0u};
            const int nc[2] = {min(kBK, a.N - pend * kBK), 0};
            ok = push(TILE_EXACT, bl, wh, nc, none, 0.f, zero2);
            pend = -1;
            if (ok) after_exact();
        }
        while (ok && gdone < gat_est) ok = push_gather();   // the rest (none if no exact tile)
        if (!dense && a.centroid && ok) {
            const int last_n = a.N - (a.nKB - 1) * kBK;
            const int nchunk = (a.nKB + kBK - 1) / kBK;
            const uint32_t *k0 = kept, *k1 = kept + a.nW, *f0 = aff, *f1 = aff + a.nW;
            auto cmask = [&](const uint32_t *k, const uint32_t *f, int cc) -> uint64_t {
                if (cc >= nchunk) return 0ull;
                const int nb = min(kBK, a.nKB - cc * kBK);
                const uint64_t valid = nb == 64 ? ~0ull : ((1ull << nb) - 1ull);
                const int w0 = 2 * cc;
                const uint64_t lo = w0 < a.nW ? (k[w0] | f[w0]) : 0u;
                const uint64_t hi = w0 + 1 < a.nW ? (k[w0 + 1] | f[w0 + 1]) : 0u;
                return valid & ~(lo | (hi << 32));
            };
            for (int cc = 0; cc < nchunk && ok; cc += 2) {
                uint64_t cm[2][2];
                int bl[2], pc[2];
                for (int x = 0; x < 2; ++x) {
                    const int c = cc + x;
                    cm[0][x] = cmask(k0, f0, c);
                    cm[1][x] = nq > 1 ? cmask(k1, f1, c) : 0ull;
                    bl[x] = c < nchunk ? c : cc;          // an empty half repeats a valid chunk
                    const int lastcol = (a.nKB - 1) - c * kBK;
                    pc[x] = (c < nchunk && last_n < kBK && lastcol >= 0 && lastcol < kBK) ? lastcol : -1;
                }
                if ((cm[0][0] | cm[0][1] | cm[1][0] | cm[1][1]) == 0ull) continue;
                const uint32_t wh[2] = {0u, 0u};
                const int nc[2] = {0, 0};
                ok = push(TILE_CENT, bl, wh, nc, pc, last_n < kBK ? log2f((float)last_n) : 0.f, cm);
            }
        }
        if (ok) {
            const int bl[2] = {0, 0};
            const uint32_t wh[2] = {0u, 0u};
            const int nc[2] = {0, 0};
            // the K side marks the end twice: at T (tile T - 2's ready, where the MMA
            // warp reads it) and at T + 1 (tile T - 1's ready, which has no K tile)
            ok = push(TILE_END, bl, wh, nc, none, 0.f, zero2);
            if (ok && is_k) ok = push(TILE_END, bl, wh, nc, none, 0.f, zero2);
        }
        if (lane == 0) {
            // no TMA write may still be in flight when the CTA exits: wait for the
            // last phase every barrier was armed with (phases complete in order; the
            // ready phases also take the softmax warps' arrivals, which every tile
            // before the end gets)
            volatile int32_t no_abort = 0;
            if (is_k) {
                for (int t = 0; t < 2 && t < j; ++t) mbar_wait(&k_full[t], 0, &no_abort, a.status, 12);
                for (int t = max(2, j - 2); t < j; ++t)
                    mbar_wait(&ready[t & 1], ((t - 2) >> 1) & 1, &no_abort, a.status, 15);
                mbar_wait(bar_q, 0, &no_abort, a.status, 14);
            } else {
                for (int s = 0; s < depth; ++s) {
                    const int n = (j - s + depth - 1) / depth;
                    if (n > 0) mbar_wait(&full[s], (n - 1) & 1, &no_abort, a.status, 12);
                }
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");   // this lane's gathered rows have landed
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issuer
        // The whole warp runs it (warp-uniform operands); one elected lane issues.
        {
            const uint32_t idesc_s = idesc_bf16_f32(kM, kTK, 0, 0);
            const uint32_t idesc_s8 = idesc_e4m3_f32(kM, kTK);
            const uint32_t idesc_o = idesc_bf16_f32(kM, D, 0, 1);
            const uint32_t idesc_o8 = idesc_e4m3_f32(kM, D) | (1u << 16);   // B (V) MN-major
            const uint32_t q_addr = smem_u32(sm + L::kOffQ);
            const uint32_t k_addr = smem_u32(sm + L::kOffK);
            const uint32_t v_addr = smem_u32(sm + L::kOffV);
            bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort_flag, a.status, 22));
            tc_fence_after();
            // rows copied by cp.async (gathers without TMA) need a proxy fence before
            // the tensor core reads them
            const bool cp_gather = a.E > 0 && !a.gather_tma;
            // Fixed order: S(0), S(1), then for each tile j the P V products of both
            // halves and S(j + 2), which goes to the buffer P(j) held (the tensor pipe
            // runs one thread's MMAs in issue order), all behind the one wait on
            // ready(j).  Every wait is a blocking try_wait: polling barriers from this
            // thread between MMAs stalls the tensor pipe.
            int T = -1;   // tile count, once the end marker is seen
            // S(ns) for a K tile that has landed (kind read after its barrier)
            auto issue_s = [&](int ns, int kind) {
                const int ks = ns % kKS;
                if (kind == TILE_END) {
                    // end-of-list marker for the softmax warps, committed at once: it
                    // completes after every MMA issued so far (P V of tiles < T - 1)
                    umma_commit_w(&s_full[ns & 1]);
                    T = ns;
                    return;
                }
                if (cp_gather && kind == TILE_GATHER) fence_async_smem();
                if (QK8) {
                    // 128 fp8 channels per 128-byte row, 32 per instruction
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk) {
                        const uint64_t ad = sdesc_sw128(q_addr + kk * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(k_addr + ks * L::kKTileBytes + kk * 32, 16, 1024);
                        umma_ss_f8_w(tmem + kColS + 128 * (ns & 1), ad, bd, idesc_s8, kk > 0 ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * (kM * 128) + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(
                            k_addr + ks * L::kKTileBytes + (kk >> 2) * (kTK * 128) + (kk & 3) * 32, 16, 1024);
                        umma_ss_w(tmem + kColS + 128 * (ns & 1), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    }
                }
                umma_commit_w(&s_full[ns & 1]);
                if (lane == 0) TRACE(2, ns);
            };
            // O_hf += P_hf(t) V_hf(t); P_h(t) is in only after the softmax warps waited
            // for V(t) (they read the tile's metadata there), so the V rows are in too
            auto issue_pv = [&](int t, int hf) {
                const int pb = t & 1, vs = t % kVS;
                if (PV8) {
                    // P as e4m3 (4 a column), V as e4m3 rows of 128 channels: K = 32 a step
#pragma unroll
                    for (int ks = 0; ks < kBK / 32; ++ks) {
                        const uint64_t bd =
                            sdesc_sw128(v_addr + vs * L::kTileBytes + hf * L::kHalfBytes + ks * 4096, 16, 1024);
                        umma_ts_f8_w(tmem + kColO + 128 * hf, tmem + kColS + 128 * pb + 64 * hf + 8 * ks, bd,
                                     idesc_o8, (t > 0 || ks > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks) {
                        const uint64_t bd =
                            sdesc_sw128(v_addr + vs * L::kTileBytes + hf * L::kHalfBytes + ks * 2048, kTK * 128, 1024);
                        umma_ts_w(tmem + kColO + 128 * hf, tmem + kColS + 128 * pb + 64 * hf + 8 * ks, bd, idesc_o,
                                  (t > 0 || ks > 0) ? 1u : 0u);
                    }
                }
            };
            for (int ns = 0; ns < 2 && ok && T < 0; ++ns) {
                ok = __all_sync(0xffffffffu, mbar_wait(&k_full[ns], 0, abort_flag, a.status, 27));
                if (!ok) break;
                tc_fence_after();
                issue_s(ns, kkind[ns]);
            }
            for (int j = 0; ok && (T < 0 || j < T); ++j) {
                ok = __all_sync(0xffffffffu, mbar_wait(&ready[j & 1], (j >> 1) & 1, abort_flag, a.status, 28));
                if (!ok) break;
                tc_fence_after();
                // the next K tile's kind, loaded before the P V issue and used after it
                const int kind2 = T < 0 ? kkind[(j + 2) % kKS] : TILE_END;
                const int vs = j % kVS;
                if (cp_gather && info[vs].h[0].x == TILE_GATHER) fence_async_smem();   // rows by cp.async
                issue_pv(j, 0);
                if (lane == 0) TRACE(3, j);
                issue_pv(j, 1);
                umma_commit_w(&v_empty[vs]);   // both halves have used the V slot
                if (T < 0) issue_s(j + 2, kind2);
            }
            umma_commit_w(bar_done);
            volatile int32_t no_abort = 0;
            mbar_wait(bar_done, 0, &no_abort, a.status, 25);
        }
    } else {
        // ---------------------------------------------------------- softmax
        // warpgroup hf owns half hf of every tile (one key block) and keeps its own
        // online softmax state and accumulator O_hf
        const int hf = warp >> 2;
        const int r = threadIdx.x & 127;                         // tile row == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int qsel = (a.Bq == 64 && !dense) ? (r >> 6) : 0;
        // fp8 Q K^T: S is in units of (Q scale of the row's 64 tokens) x (K scale of the half)
        const float scale_q =
            QK8 ? a.scale_log2 * a.sq8[(int64_t)bh * a.nb64 + min(row0 + r, a.N - 1) / 64] : a.scale_log2;
        const uint32_t col_o = kColO + 128 * hf;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        int j = 0;
        for (;; ++j) {
            const int vs = j % kVS;
            const TileInfo *ti = const_cast<const TileInfo *>(info) + vs;
            // S(j) and V(j) are usually in by now: test both and load this half's
            // metadata in one go (one shared-memory round trip); else wait and reload
            int4 hq;
            if (!__all_sync(0xffffffffu, test2_load16(&s_full[j & 1], (j >> 1) & 1, &v_full[vs], (j / kVS) & 1,
                                                      &ti->h[hf], hq))) {
                ok = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag, a.status, 30) &&
                     mbar_wait(&v_full[vs], (j / kVS) & 1, abort_flag, a.status, 31);
                if (!(ok = __all_sync(0xffffffffu, ok))) break;
                hq = ti->h[hf];   // (a plain load: the waits above order it)
            }
            tc_fence_after();
            const int kind = hq.x;
            if (kind == TILE_END) break;
            const float scale = QK8 ? scale_q * ti->ksc[hf] : scale_q;
            if (r == 0) TRACE(4 + 3 * hf, j);
            float s[64];
            const uint32_t col_s = kColS + 128 * (j & 1) + 64 * hf;   // this half's S, then its P
            tmem_ld32(tmem + lane_base + col_s, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
            tmem_ld32(tmem + lane_base + col_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
            tmem_ld_wait();
            if (r == 0) TRACE(5 + 3 * hf, j);

            // 0: skip (no active column), 1: all 64 columns active, 2: masked / biased
            int mode;
            if (kind == TILE_EXACT) {
                const bool act = ((uint32_t)hq.y >> qsel) & 1u;
                const int nc = act ? hq.z : 0;
                if (nc >= kBK) {
                    mode = 1;
                } else if (nc <= 0) {
                    mode = 0;
                } else {
                    mode = 2;
                    const float2 sc2 = make_float2(scale, scale);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float2 y = fmul2(make_float2(s[2 * c], s[2 * c + 1]), sc2);
                        s[2 * c] = 2 * c < nc ? y.x : -INFINITY;
                        s[2 * c + 1] = 2 * c + 1 < nc ? y.y : -INFINITY;
                    }
                }
            } else if (kind == TILE_CENT) {
                const uint64_t msk = ti->cmask[qsel][hf];
                const int pc = hq.w;
                const float pbias = ti->last_bias;
                mode = msk ? 2 : 0;
                if (msk) {
                    const float2 sc2 = make_float2(scale, scale);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        // log2(64) for full blocks
                        const float2 b2 = make_float2(2 * c == pc ? pbias : 6.0f, 2 * c + 1 == pc ? pbias : 6.0f);
                        const float2 y = ffma2(make_float2(s[2 * c], s[2 * c + 1]), sc2, b2);
                        s[2 * c] = ((msk >> (2 * c)) & 1ull) ? y.x : -INFINITY;
                        s[2 * c + 1] = ((msk >> (2 * c + 1)) & 1ull) ? y.y : -INFINITY;
                    }
                }
            } else {
                // gathered columns: extra tokens (bias 0) and modified centroids
                // (bias log2 of their remaining token count)
                const uint64_t msk = ti->cmask[qsel][hf];
                const float *bias = bias_sm + vs * kTK + 64 * hf;
                mode = msk ? 2 : 0;
                if (msk) {
                    const float2 sc2 = make_float2(scale, scale);
                    const float2 *bias2 = reinterpret_cast<const float2 *>(bias);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float2 y = ffma2(make_float2(s[2 * c], s[2 * c + 1]), sc2, bias2[c]);
                        s[2 * c] = ((msk >> (2 * c)) & 1ull) ? y.x : -INFINITY;
                        s[2 * c + 1] = ((msk >> (2 * c + 1)) & 1ull) ? y.y : -INFINITY;
                    }
                }
            }
            uint32_t pk[32];
            bool rescale = false;
            float alpha = 1.f;
            if (mode == 0) {
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = 0u;
            } else {
                // P = 2^(x - m_ref) with a lazily raised reference m_ref.  With bf16 P
                // the tile's maximum is skipped once m_ref is set: every p is at most
                // the tile's sum, so a sum within kOptSum proves the tile fits (bf16 P
                // and the f32 sums keep the same relative precision at any scale, which
                // cancels in O / l).  A larger sum -- the row's maximum rose by more
                // than about log2(kOptSum / 64) -- takes the maximum and the rescale,
                // as does every tile with e4m3 P (at most 448).
                bool exact = PV8 || m_ref == -INFINITY;
                float lt;
                for (;;) {
                    if (exact) {
                        const float mt = mode == 1 ? max64(s) * scale : max64(s);
                        if (mt > m_ref) {
                            if (m_ref == -INFINITY) {
                                m_ref = mt;
                            } else if (mt > m_ref + kRescaleLog2) {
                                alpha = ex2(m_ref - mt);
                                l *= alpha;
                                m_ref = mt;
                                rescale = true;
                            }
                        }
                    }
                    const float mref = m_ref == -INFINITY ? 0.f : m_ref;
                    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    const float2 nm2 = make_float2(-mref, -mref);
                    if (mode == 1) {
                        const float2 sc2 = make_float2(scale, scale);
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const float2 x = ffma2(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
                            const float p0 = ex2(x.x), p1 = ex2(x.y);
                            acc[c & 1] = fadd2(acc[c & 1], make_float2(p0, p1));
                            pk[c] = PV8 ? (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3)
                                        : pack_bf16x2(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const float2 x = fadd2(make_float2(s[2 * c], s[2 * c + 1]), nm2);
                            const float p0 = ex2(x.x), p1 = ex2(x.y);
                            acc[c & 1] = fadd2(acc[c & 1], make_float2(p0, p1));
                            pk[c] = PV8 ? (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3)
                                        : pack_bf16x2(p0, p1);
                        }
                    }
                    lt = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
                    if (exact || lt <= kOptSum) break;   // (a NaN sum takes the exact pass)
                    exact = true;
                }
                l += lt;
            }
            if (r == 0) TRACE(10 + 3 * hf, j);
            if (r == 0) TRACE(11 + 3 * hf, j);
            if constexpr (PV8) {
                // e4m3 P: four a column (the row sum l keeps the unrounded values)
                uint32_t pk8[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk8[i] = (pk[2 * i] & 0xffffu) | (pk[2 * i + 1] << 16);
                tmem_st16(tmem + lane_base + col_s, pk8);
            } else {
                tmem_st32(tmem + lane_base + col_s, pk);   // over this half's S, already read
            }
            if (__any_sync(0xffffffffu, rescale)) {
                // the accumulator must hold every earlier P V product before it is scaled
                // (S(j + 1), or the end marker, is issued after P V(j - 1))
                ok = mbar_wait(&s_full[(j + 1) & 1], ((j + 1) >> 1) & 1, abort_flag, a.status, 33);
                if (!(ok = __all_sync(0xffffffffu, ok))) break;
                tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + col_o + cc * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tmem + lane_base + col_o + cc * 32, o);
                }
            }
            tmem_st_wait();
            if (r == 0) TRACE(12 + 3 * hf, j);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[j & 1]);
            if (r == 0) TRACE(6 + 3 * hf, j);
        }
        const int T = j;
        if (ok && T >= 1) ok = mbar_wait(bar_done, 0, abort_flag, a.status, 34);   // every MMA done
        ok = __all_sync(0xffffffffu, ok);
        // ------------------------------------------------------ epilogue
        // merge the halves: O = (wA O_A + wB O_B) / (wA lA + wB lB), w = 2^(m_half - m)
        const bool have = T >= 1 && l > 0.f;
        ml[hf * kM + r] = make_float2(have ? m_ref : -INFINITY, have ? l : 0.f);
        named_bar(1, 256);
        const float2 A = ml[r], Bv = ml[kM + r];
        const float m = fmaxf(A.x, Bv.x);
        const float wA = A.x > -INFINITY ? ex2(A.x - m) : 0.f;
        const float wB = Bv.x > -INFINITY ? ex2(Bv.x - m) : 0.f;
        const float lt = wA * A.y + wB * Bv.y;
        tc_fence_after();
        if (ok) {
            const bool row_ok = r < nvalid;
            const int n = row0 + r;
            const bool split = dense && a.dense_split > 1;
            // a sparse item leaves rows of the dense range to the dense items
            const bool mine = row_ok && (dense || n < a.dense_begin || n >= a.dense_end);
            const float inv = split ? 1.f : (lt > 0.f ? 1.f / lt : 0.f);
            const float cA = wA * inv, cB = wB * inv;
#pragma unroll 1
            for (int cc = hf * (D / 64); cc < (hf + 1) * (D / 64); ++cc) {
                uint32_t oa[32], ob[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + kColO + cc * 32, oa);
                tmem_ld32(tmem + lane_base + kColO + 128 + cc * 32, ob);
                tmem_ld_wait();
                if (!(split ? row_ok : mine)) continue;
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float xa = cA > 0.f ? cA * __uint_as_float(oa[e]) : 0.f;
                    const float xb = cB > 0.f ? cB * __uint_as_float(ob[e]) : 0.f;
                    v[e] = xa + xb;
                }
                if constexpr (PV8) {
                    // V was stored divided by its channel's scale
                    const float4 *sv4 = reinterpret_cast<const float4 *>(a.sv8 + (int64_t)bh * D + cc * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 s4 = __ldg(sv4 + e);
                        v[4 * e] *= s4.x;
                        v[4 * e + 1] *= s4.y;
                        v[4 * e + 2] *= s4.z;
                        v[4 * e + 3] *= s4.w;
                    }
                }
                if (split) {
                    // unnormalised partial in the frame of m, merged by combine_kernel
                    float4 *dst = reinterpret_cast<float4 *>(a.part_o + (pidx * kM + r) * D + cc * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
                    continue;
                }
                const int64_t off = (int64_t)b * a.sb + (int64_t)pos_token(a, n) * a.sn + (int64_t)h * a.sh + cc * 32;
                if (a.out_f32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + off);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + off);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pack_bf16x2(v[8 * e], v[8 * e + 1]), pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                                            pack_bf16x2(v[8 * e + 4], v[8 * e + 5]),
                                            pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
                }
            }
            if (hf == 0) {
                if (split) {
                    float *pm = a.part_ml + (pidx * kM + r) * 2;
                    pm[0] = lt > 0.f ? m : -INFINITY;
                    pm[1] = lt;
                } else if (mine && a.lse != nullptr) {
                    a.lse[(int64_t)bh * a.N + pos_token(a, n)] =
                        lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
#ifdef BSA_TRACE
    {
        const int c = (int)blockIdx.x - a.trace_base;
        if (a.trace != nullptr && c >= 0 && c < kTraceCtas)
            for (int i = threadIdx.x; i < kTraceTiles * kTraceEvents; i += blockDim.x)
                a.trace[(int64_t)c * kTraceTiles * kTraceEvents + i] = trace_sm[i];
    }
#endif
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge the key-chunk partials of the dense rows: one thread per row.
__global__ void __launch_bounds__(128) combine_kernel(AttnArgs a, int d)
{
    const int64_t tt = blockIdx.x;                 // (bh, tile)
    const int r = threadIdx.x;
    const int t = (int)(tt % a.n_dense);
    const int bh = (int)(tt / a.n_dense);
    const int b = bh / a.H, h = bh % a.H;
    const int n = a.dense_begin + t * kM + r;
    if (n >= a.dense_end) return;
    const int S = a.dense_split;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, a.part_ml[((tt * S + s) * kM + r) * 2]);
    float l = 0.f;
    for (int s = 0; s < S; ++s) {
        const float *ml = a.part_ml + ((tt * S + s) * kM + r) * 2;
        if (ml[0] > -INFINITY) l += ml[1] * exp2f(ml[0] - m);
    }
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const int64_t off = (int64_t)b * a.sb + (int64_t)n * a.sn + (int64_t)h * a.sh;
    for (int c0 = 0; c0 < d; c0 += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < S; ++s) {
            const float ms = a.part_ml[((tt * S + s) * kM + r) * 2];
            if (!(ms > -INFINITY)) continue;
            const float w = exp2f(ms - m) * inv_l;
            const float4 o = *reinterpret_cast<const float4 *>(a.part_o + ((tt * S + s) * kM + r) * d + c0);
            acc.x += w * o.x;
            acc.y += w * o.y;
            acc.z += w * o.z;
            acc.w += w * o.w;
        }
        if (a.out_f32) {
            *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + off + c0) = acc;
        } else {
            uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.out) + off + c0) = pk;
        }
    }
    if (a.lse != nullptr)
        a.lse[(int64_t)bh * a.N + n] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

template <int CPL>
__device__ __forceinline__ void load_bf16_vec(const __nv_bfloat16 *p, float (&f)[CPL])
{
    if constexpr (CPL == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        f[0] = __uint_as_float(w.x << 16);
        f[1] = __uint_as_float(w.x & 0xffff0000u);
        f[2] = __uint_as_float(w.y << 16);
        f[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(p));
        f[0] = __uint_as_float(w << 16);
        f[1] = __uint_as_float(w & 0xffff0000u);
    }
}

// Modified centroids of the blocks that gave extra tokens: for query block r and
// a block b that gave e of its n tokens to r's list and keeps some, the centroid
// of its remaining tokens, (n kbar_b - sum of the extra keys) / (n - e), with
// bias log2(n - e); the same for V.  Row r's entries, in ascending block order,
// are numbered idx = xoff[r] .. xoff[r] + xcnt[r] - 1 (as many as the capacity
// holds); the centroids themselves are stored grouped by source block, entry
// idx at slot[idx].  Steps: count each row's entries (mc_count_kernel) and scan;
// per (b, h) and group of query blocks, count the entries that fit per source
// block and scan (mc_group_kernel<1>), then list them (mc_group_kernel<2>), with
// counters in shared memory; form each block's entries from its K and V rows,
// read once into shared memory (mc_build_kernel).

struct McArgs {
    const int32_t *extra_idx, *extra_count;
    int64_t rows;
    int H, N, nQB, nKB, E;
    int G, rpg;                  // query-block groups per (b, h), query blocks per group
    int32_t *xcnt;
    const int64_t *xoff;
    int32_t *cnt3;               // [B*H, nKB, G] entries that fit, per (source block, group)
    const int64_t *off3;         // [B*H*nKB*G + 1] its exclusive scan
    uint64_t *ent;               // [cap] left-out tokens of each entry (bit t: token 64 b + t), by block
    int32_t *slot;               // [cap] where entry idx sits in ent and in the centroid arrays
    float *xbias;                // [cap] by idx
    int64_t cap;
    int32_t *status;
};

// Walks row r's ascending extra-token list (one warp; E <= 256, so 8 tokens a
// lane, all loaded at once) by runs of tokens from one block, in token order:
// f(blk, mask, e, rank) once per run, on one lane, rank = the run's place among
// the row's runs whose block keeps tokens (-1 for a run that takes the whole
// block).  In each 32-token chunk a run starts where the block changes (one
// ballot); its tokens' bits are OR-ed into its first lane by a segmented
// shuffle-down; a run that reaches the chunk's last lane and goes on in the next
// chunk is carried over.  A token outside [0, N) belongs to no run (it is
// reported).  Returns the count of ranked runs.
template <typename F>
__device__ __forceinline__ int walk_runs(const McArgs &a, int64_t r, int lane, F &&f)
{
    static_assert(kMaxE == 256, "8 tokens per lane");
    const int n = min(a.extra_count[r], a.E);
    const int32_t *ex = a.extra_idx + r * a.E;
    int tk[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int i = 32 * u + lane;
        tk[u] = i < n ? ex[i] : -1;
        if (i < n && (tk[u] < 0 || tk[u] >= a.N)) {
            report(a.status, BSA_DEV_INTERNAL, 3);
            tk[u] = -1;
        }
    }
    int ranked = 0;
    int cblk = -1, ce = 0;   // the run carried over from the previous chunk
    uint64_t cmask = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        if (32 * u >= n) break;
        const int tok = tk[u];
        const int blk = tok >= 0 ? tok >> 6 : -1 - lane;   // lanes without a token stand alone
        const int prev = __shfl_up_sync(0xffffffffu, blk, 1);
        const uint32_t bnd = __ballot_sync(0xffffffffu, lane == 0 || blk != prev);
        const uint32_t above = bnd & ~((2u << lane) - 1u);   // (2u << 31 wraps to 0: all ones)
        const int end = above ? __ffs(above) - 2 : 31;       // last lane of this lane's run
        const int o = tok & 63;
        uint32_t lo = tok >= 0 && o < 32 ? 1u << o : 0u, hi = tok >= 0 && o >= 32 ? 1u << (o - 32) : 0u;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t vlo = __shfl_down_sync(0xffffffffu, lo, off);
            const uint32_t vhi = __shfl_down_sync(0xffffffffu, hi, off);
            if (lane + off <= end) {
                lo |= vlo;
                hi |= vhi;
            }
        }
        const bool first = (bnd >> lane) & 1u;
        uint64_t mask = ((uint64_t)hi << 32) | lo;
        int e = end - lane + 1;
        if (lane == 0 && blk == cblk) {
            e += ce;
            mask |= cmask;
        }
        const int nxt = u < 7 ? __shfl_sync(0xffffffffu, tk[u < 7 ? u + 1 : u], 0) : -1;
        const bool cont = tok >= 0 && end == 31 && nxt >= 0 && (nxt >> 6) == blk;
        const bool emit = tok >= 0 && first && !cont;
        const bool keeps = emit && min(64, a.N - blk * 64) - e > 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, keeps);
        if (emit) f(blk, mask, e, keeps ? ranked + __popc(bal & ((1u << lane) - 1u)) : -1);
        ranked += __popc(bal);
        const uint32_t cl = __ballot_sync(0xffffffffu, cont && first);
        if (cl) {
            const int src = __ffs(cl) - 1;
            cblk = __shfl_sync(0xffffffffu, blk, src);
            ce = __shfl_sync(0xffffffffu, e, src);
            cmask = __shfl_sync(0xffffffffu, mask, src);
        } else {
            cblk = -1;
            ce = 0;
            cmask = 0;
        }
    }
    return ranked;
}

// Each row's entry count (one warp per row).
__global__ void __launch_bounds__(256) mc_count_kernel(McArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= a.rows) return;
    const int cnt = walk_runs(a, r, lane, [](int, uint64_t, int, int) {});
    if (lane == 0) a.xcnt[r] = cnt;
}

// One CTA per ((b, h), group g of query blocks), a warp per row, one counter per
// source block in shared memory.  kMode 1: the entries that fit, per source
// block, into cnt3; 2: list them -- ent and slot from the scanned counts, the
// biases -- and cut each row's count to what fits.
template <int kMode>
__global__ void __launch_bounds__(256) mc_group_kernel(McArgs a)
{
    extern __shared__ int32_t cs[];   // [nKB]
    const int64_t bh = blockIdx.x / a.G;
    const int g = (int)(blockIdx.x % a.G);
    const int i0 = g * a.rpg, i1 = min(a.nQB, i0 + a.rpg);
    const int64_t b3 = bh * a.nKB;
    for (int blk = threadIdx.x; blk < a.nKB; blk += blockDim.x)
        cs[blk] = kMode == 1 ? 0 : (int32_t)a.off3[(b3 + blk) * a.G + g];
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = i0 + warp; i < i1; i += (int)(blockDim.x >> 5)) {
        const int64_t r = bh * a.nQB + i;
        const int64_t x0 = a.xoff[r];
        const int cnt = walk_runs(a, r, lane, [&](int blk, uint64_t mask, int e, int rank) {
            if (rank < 0 || x0 + rank >= a.cap) return;
            if (kMode == 1) {
                atomicAdd(&cs[blk], 1);
            } else {
                const int sl = atomicAdd(&cs[blk], 1);
                a.ent[sl] = mask;
                a.slot[x0 + rank] = sl;
                a.xbias[x0 + rank] = log2f((float)(min(64, a.N - blk * 64) - e));
            }
        });
        if (kMode == 2 && lane == 0) {
            const int64_t fit = a.cap - x0;
            const int kept = (int)(fit < 0 ? 0 : (fit < cnt ? fit : cnt));
            a.xcnt[r] = kept;
            if (kept < cnt) report(a.status, BSA_DEV_CAPACITY, 2);
        }
    }
    if (kMode == 1) {
        __syncthreads();
        for (int blk = threadIdx.x; blk < a.nKB; blk += blockDim.x) a.cnt3[(b3 + blk) * a.G + g] = cs[blk];
    }
}

// One CTA per (source block, b, h) -- the heads of one block side by side, so
// that CTAs running together read neighbouring parts of the same token rows --
// and 2 d threads.  The block's K and V rows go to shared memory once; then each
// entry listed under the block is formed by 2 d / 8 lanes, a lane owning 8
// channels of K or of V: in f32, the block's sum n kbar_b minus its left-out
// tokens in token order, times 1/(n - e), rounded to bf16, written at the entry's
// slot (a block's slots are consecutive).
template <int D>
__global__ void __launch_bounds__(2 * D) mc_build_kernel(McArgs a, const float *__restrict__ kbar,
                                                         const float *__restrict__ vbar,
                                                         const __nv_bfloat16 *__restrict__ k,
                                                         const __nv_bfloat16 *__restrict__ v, int64_t sb, int64_t sn,
                                                         int64_t sh, __nv_bfloat16 *__restrict__ xk,
                                                         __nv_bfloat16 *__restrict__ xv)
{
    constexpr int kThr = 2 * D;
    constexpr int kCpr = D / 8;                 // 16-byte chunks per row
    constexpr int kLpe = 2 * kCpr;              // lanes per entry
    constexpr int kEpw = 32 / kLpe;             // entries per warp at a time
    constexpr int kWarps = kThr / 32;
    __shared__ __align__(16) __nv_bfloat16 rows_s[2][64][D];
    __shared__ uint64_t es[kThr];
    __shared__ float rinv[65];
    const int64_t BH = a.rows / a.nQB;
    const int blk = (int)(blockIdx.x / BH);
    const int64_t bh = blockIdx.x % BH;
    const int64_t e0 = a.off3[(bh * a.nKB + blk) * a.G];
    const int n_ent = (int)(a.off3[(bh * a.nKB + blk + 1) * a.G] - e0);
    if (n_ent == 0) return;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const int nb = min(64, a.N - blk * 64);
    // 2 tensors x 64 rows x kCpr chunks = 8 per thread, all in flight at once
    uint4 ld[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int x = threadIdx.x + kThr * u;
        const int t = x / (64 * kCpr), row = (x / kCpr) % 64, c16 = x % kCpr;
        const __nv_bfloat16 *src = (t ? v : k) + (int64_t)b * sb + (int64_t)(blk * 64 + row) * sn +
                                   (int64_t)h * sh + c16 * 8;
        if (row < nb) ld[u] = __ldg(reinterpret_cast<const uint4 *>(src));
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int x = threadIdx.x + kThr * u;
        const int t = x / (64 * kCpr), row = (x / kCpr) % 64, c16 = x % kCpr;
        if (row < nb) *reinterpret_cast<uint4 *>(&rows_s[t][row][c16 * 8]) = ld[u];
    }
    if (threadIdx.x <= 64) rinv[threadIdx.x] = threadIdx.x > 0 ? 1.f / (float)threadIdx.x : 0.f;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / kLpe, l = lane % kLpe;
    const int t = l / kCpr, c0 = (l % kCpr) * 8;
    float2 base[4];
    {
        const float4 *m = reinterpret_cast<const float4 *>((t ? vbar : kbar) + (bh * a.nKB + blk) * D + c0);
        const float4 m0 = m[0], m1 = m[1];
        const float fn = (float)nb;
        base[0] = make_float2(fn * m0.x, fn * m0.y);
        base[1] = make_float2(fn * m0.z, fn * m0.w);
        base[2] = make_float2(fn * m1.x, fn * m1.y);
        base[3] = make_float2(fn * m1.z, fn * m1.w);
    }
    __nv_bfloat16 *dst = (t ? xv : xk) + e0 * D + c0;
    for (int i0 = 0; i0 < n_ent; i0 += kThr) {
        __syncthreads();   // (the first also publishes the rows and rinv)
        if (i0 + (int)threadIdx.x < n_ent) es[threadIdx.x] = a.ent[e0 + i0 + threadIdx.x];
        __syncthreads();
        const int m = min(kThr, n_ent - i0);
        for (int i = warp * kEpw + sub; i < m; i += kWarps * kEpw) {
            const uint64_t em = es[i];
            float2 sum[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) sum[j] = base[j];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t mk = (uint32_t)(em >> (32 * half));
                while (mk) {
                    const int bit = 32 * half + __ffs(mk) - 1;
                    mk &= mk - 1;
                    const uint4 w = *reinterpret_cast<const uint4 *>(&rows_s[t][bit][c0]);
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        sum[j] = fsub2(sum[j], make_float2(__uint_as_float(wv[j] << 16),
                                                           __uint_as_float(wv[j] & 0xffff0000u)));
                }
            }
            const float ri = rinv[nb - __popcll(em)];
            const float2 r2 = make_float2(ri, ri);
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 y = fmul2(sum[j], r2);
                o[j] = pack_bf16x2(y.x, y.y);
            }
            *reinterpret_cast<uint4 *>(dst + (int64_t)(i0 + i) * D) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Per sparse tile of the fine pass (query blocks qb0 and qb0 + 1 for 64-row
// blocks, one 128-row block otherwise): the union of its query blocks' ascending
// extra-token lists, an entry being the token with bit 30 set if the first query
// block chose it and bit 31 if the second did; padded to a multiple of 4 with
// repeats of its last token (no bit set) so that a gather of 4 rows never mixes
// tokens with modified centroids.  One warp per tile.  Union rank of a token of
// one list = its index + the other list's tokens below it - those of them that
// both lists hold.
__global__ void __launch_bounds__(128) glist_kernel(const int32_t *__restrict__ extra_idx,
                                                    const int32_t *__restrict__ extra_count, int E, int nQB, int Bq,
                                                    int n_sparse, int64_t ntiles, uint32_t *__restrict__ glist,
                                                    int32_t *__restrict__ glcnt)
{
    __shared__ int32_t sA[4][kMaxE], sB[4][kMaxE], lbA[4][kMaxE], lbB[4][kMaxE], PA[4][kMaxE + 1],
        PB[4][kMaxE + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 4 + warp;
    if (t >= ntiles) return;
    const int64_t bh = t / n_sparse;
    const int qb0 = (int)((t % n_sparse) * kM / Bq);
    const int nq = (Bq == 64 && qb0 + 1 < nQB) ? 2 : 1;
    const int64_t r0 = bh * nQB + qb0;
    const int n0 = min(extra_count[r0], E), n1 = nq > 1 ? min(extra_count[r0 + 1], E) : 0;
    int32_t *A = sA[warp], *B = sB[warp];
    {
        // both lists, every load in flight before the first store
        int va[kMaxE / 32], vb[kMaxE / 32];
#pragma unroll
        for (int u = 0; u < kMaxE / 32; ++u) {
            const int i = 32 * u + lane;
            va[u] = i < n0 ? extra_idx[r0 * E + i] : 0;
            vb[u] = i < n1 ? extra_idx[(r0 + 1) * E + i] : 0;
        }
#pragma unroll
        for (int u = 0; u < kMaxE / 32; ++u) {
            const int i = 32 * u + lane;
            if (i < n0) A[i] = va[u];
            if (i < n1) B[i] = vb[u];
        }
    }
    __syncwarp();
    auto lower_bound = [](const int32_t *X, int n, int key) {
        int lo = 0, hi = n;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (X[mid] < key)
                lo = mid + 1;
            else
                hi = mid;
        }
        return lo;
    };
    for (int i = lane; i < n0; i += 32) {
        const int lb = lower_bound(B, n1, A[i]);
        lbA[warp][i] = lb | ((lb < n1 && B[lb] == A[i]) ? 0x40000000 : 0);
    }
    for (int i = lane; i < n1; i += 32) {
        const int lb = lower_bound(A, n0, B[i]);
        lbB[warp][i] = lb | ((lb < n0 && A[lb] == B[i]) ? 0x40000000 : 0);
    }
    __syncwarp();
    // P[k] = entries of a list among its first k that the other list holds too
    auto prefix = [&](const int32_t *lb, int n, int32_t *P) {
        int carry = 0;
        for (int k0 = 0; k0 <= n; k0 += 32) {
            const int k = k0 + lane;
            int x = (k > 0 && k <= n) ? ((lb[k - 1] >> 30) & 1) : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (k <= n) P[k] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    };
    prefix(lbA[warp], n0, PA[warp]);
    prefix(lbB[warp], n1, PB[warp]);
    __syncwarp();
    uint32_t *out = glist + t * kGlistCap;
    for (int i = lane; i < n0; i += 32) {
        const int v = lbA[warp][i], lb = v & 0x3fffffff;
        const bool both = (v >> 30) & 1;
        out[i + lb - PB[warp][lb]] = (uint32_t)A[i] | (both ? 0xC0000000u : 0x40000000u);
    }
    for (int i = lane; i < n1; i += 32) {
        const int v = lbB[warp][i], lb = v & 0x3fffffff;
        if ((v >> 30) & 1) continue;   // listed with the first query block
        out[i + lb - PA[warp][lb]] = (uint32_t)B[i] | 0x80000000u;
    }
    const int U0 = n0 + n1 - PA[warp][n0], U = (U0 + 3) & ~3;
    __syncwarp();
    if (lane < U - U0) out[U0 + lane] = out[U0 - 1] & 0x3fffffffu;
    if (lane == 0) glcnt[t] = U;
}

// bf16 copies of f32 centroids: elementwise, grid-stride.
__global__ void to_bf16_kernel(const float *__restrict__ src, __nv_bfloat16 *__restrict__ dst, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

// f32 [B, N, H, d] strided -> bf16 contiguous [B, N, H, d].
__global__ void inputs_to_bf16_kernel(const float *__restrict__ src, __nv_bfloat16 *__restrict__ dst,
                                      int B, int N, int H, int d, int64_t sb, int64_t sn, int64_t sh)
{
    const int64_t total = (int64_t)B * N * H * d;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % d);
        const int64_t t = i / d;
        const int hh = (int)(t % H);
        const int64_t t2 = t / H;
        const int n = (int)(t2 % N);
        const int bb = (int)(t2 / N);
        dst[i] = __float2bfloat16_rn(src[(int64_t)bb * sb + (int64_t)n * sn + (int64_t)hh * sh + c]);
    }
}

// ------------------------------------------------------------------ fp8 Q K^T

// e4m3 copy of 64 rows of one head ([B, N, H, 128] bf16 in, contiguous
// [B, N, H, 128] fp8 out) with one scale per (b, h, 64-token block): the
// block's largest |x| maps to 448, the largest finite e4m3 value (scale 1
// for an all-zero block); x8 = round-to-nearest(x / scale), saturating.
// One CTA per (b * H + h, block); thread t: row t / 4, channels 32 (t % 4) ...
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16 *__restrict__ src, int64_t sb,
                                                         int64_t sn, int64_t sh, int N, int H, int nb64,
                                                         uint8_t *__restrict__ dst, float *__restrict__ scale)
{
    __shared__ float wmax[8];
    const int64_t bh = blockIdx.y;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int blk = blockIdx.x;
    const int row = threadIdx.x >> 2, c0 = 32 * (threadIdx.x & 3);
    const int n = blk * 64 + row;
    float x[32];
    if (n < N) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src + (int64_t)b * sb + (int64_t)n * sn + (int64_t)h * sh + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 w = p[i];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[8 * i + 2 * e] = __uint_as_float(ww[e] << 16);
                x[8 * i + 2 * e + 1] = __uint_as_float(ww[e] & 0xffff0000u);
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
    }
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    m = wmax[0];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
    const float sc = m > 0.f ? m / 448.f : 1.f;
    const float inv = 1.f / sc;
    if (threadIdx.x == 0) scale[bh * nb64 + blk] = sc;
    if (n >= N) return;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i] * inv, x[4 * i + 1] * inv),
                                                                 __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(x[4 * i + 2] * inv, x[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
        pk[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    uint4 *o = reinterpret_cast<uint4 *>(dst + (((int64_t)b * N + n) * H + h) * 128 + c0);
    o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// e4m3 centroids [BH, nKB, 128] from the f32 means, one scale per 64 centroids.
__global__ void __launch_bounds__(256) quant_cent_kernel(const float *__restrict__ kbar, int nKB, int nch,
                                                         uint8_t *__restrict__ dst, float *__restrict__ scale)
{
    __shared__ float wmax[8];
    const int64_t bh = blockIdx.y;
    const int ch = blockIdx.x;
    const int row = threadIdx.x >> 2, c0 = 32 * (threadIdx.x & 3);
    const int j = ch * 64 + row;
    float x[32];
    if (j < nKB) {
        const float4 *p = reinterpret_cast<const float4 *>(kbar + ((int64_t)bh * nKB + j) * 128 + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 v = p[i];
            x[4 * i] = v.x;
            x[4 * i + 1] = v.y;
            x[4 * i + 2] = v.z;
            x[4 * i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
    }
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    m = wmax[0];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
    const float sc = m > 0.f ? m / 448.f : 1.f;
    const float inv = 1.f / sc;
    if (threadIdx.x == 0) scale[bh * nch + ch] = sc;
    if (j >= nKB) return;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i] * inv, x[4 * i + 1] * inv),
                                                                 __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(x[4 * i + 2] * inv, x[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
        pk[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    uint4 *o = reinterpret_cast<uint4 *>(dst + ((int64_t)bh * nKB + j) * 128 + c0);
    o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// ------------------------------------------------------------------ fp8 P V

// Largest |v| per (b, h, channel) of V, as the bits of a non-negative float
// (atomicMax on them orders like the floats; bits zeroed beforehand).  One CTA
// per (b * H + h, 256 tokens); thread t: channel t % 128, tokens of half t / 128.
__global__ void __launch_bounds__(256) vmax_kernel(const __nv_bfloat16 *__restrict__ v, int64_t sb, int64_t sn,
                                                   int64_t sh, int N, int H, uint32_t *__restrict__ maxbits)
{
    __shared__ float part[256];
    const int64_t bh = blockIdx.y;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int c = threadIdx.x & 127, half = threadIdx.x >> 7;
    const int n0 = blockIdx.x * 256 + half * 128, n1 = min(N, n0 + 128);
    const __nv_bfloat16 *base = v + (int64_t)b * sb + (int64_t)h * sh + c;
    float m = 0.f;
    for (int n = n0; n < n1; ++n) m = fmaxf(m, fabsf(__bfloat162float(base[(int64_t)n * sn])));
    part[threadIdx.x] = m;
    __syncthreads();
    if (half == 0) atomicMax(&maxbits[bh * 128 + c], __float_as_uint(fmaxf(m, part[threadIdx.x + 128])));
}

// In place: the largest |v| of each channel -> its scale (largest / 448; 1 for
// an all-zero channel).
__global__ void sv_scale_kernel(uint32_t *__restrict__ sv, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float m = __uint_as_float(sv[i]);
        sv[i] = __float_as_uint(m > 0.f ? m / 448.f : 1.f);
    }
}

// e4m3 copy of V ([B, N, H, 128] bf16 in, contiguous [B, N, H, 128] e4m3 out),
// x8 = round-to-nearest(x / scale of its channel), saturating.  One CTA per
// (b * H + h, 64 tokens); thread t: row t / 4, channels 32 (t % 4) ...
__global__ void __launch_bounds__(256) quant_v_kernel(const __nv_bfloat16 *__restrict__ src, int64_t sb, int64_t sn,
                                                      int64_t sh, int N, int H, const float *__restrict__ sv,
                                                      uint8_t *__restrict__ dst)
{
    const int64_t bh = blockIdx.y;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int row = threadIdx.x >> 2, c0 = 32 * (threadIdx.x & 3);
    const int n = blockIdx.x * 64 + row;
    if (n >= N) return;
    const uint4 *p = reinterpret_cast<const uint4 *>(src + (int64_t)b * sb + (int64_t)n * sn + (int64_t)h * sh + c0);
    const float *s = sv + bh * 128 + c0;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = p[i];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        float x[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[2 * e] = __uint_as_float(ww[e] << 16) / s[8 * i + 2 * e];
            x[2 * e + 1] = __uint_as_float(ww[e] & 0xffff0000u) / s[8 * i + 2 * e + 1];
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const __nv_fp8x2_storage_t lo =
                __nv_cvt_float2_to_fp8x2(make_float2(x[4 * e], x[4 * e + 1]), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t hi =
                __nv_cvt_float2_to_fp8x2(make_float2(x[4 * e + 2], x[4 * e + 3]), __NV_SATFINITE, __NV_E4M3);
            pk[2 * i + e] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
    }
    uint4 *o = reinterpret_cast<uint4 *>(dst + (((int64_t)b * N + n) * H + h) * 128 + c0);
    o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// e4m3 value centroids [BH, nKB, 128] from the f32 means, with the channel scales of V.
__global__ void __launch_bounds__(256) quant_vcent_kernel(const float *__restrict__ vbar, int nKB,
                                                          const float *__restrict__ sv, uint8_t *__restrict__ dst)
{
    const int64_t bh = blockIdx.y;
    const int row = threadIdx.x >> 2, c0 = 32 * (threadIdx.x & 3);
    const int j = blockIdx.x * 64 + row;
    if (j >= nKB) return;
    const float4 *p = reinterpret_cast<const float4 *>(vbar + ((int64_t)bh * nKB + j) * 128 + c0);
    const float *s = sv + bh * 128 + c0;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 v = p[i];
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
            make_float2(v.x / s[4 * i], v.y / s[4 * i + 1]), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(v.z / s[4 * i + 2], v.w / s[4 * i + 3]), __NV_SATFINITE, __NV_E4M3);
        pk[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    uint4 *o = reinterpret_cast<uint4 *>(dst + ((int64_t)bh * nKB + j) * 128 + c0);
    o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
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

// bf16 [B, N, H, d] with element strides; box = 64 channels x 1 head x rows tokens x 1.
bool make_map_bnhd(CUtensorMap *m, const void *base, int B, int N, int H, int d, int64_t sb, int64_t sn,
                   int64_t sh, int rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)sh * 2, (cuuint64_t)sn * 2, (cuuint64_t)sb * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bytes (fp8) [B, N, H, d] contiguous; box = 128 channels x 1 head x rows tokens x 1.
bool make_map_u8_bnhd(CUtensorMap *m, const void *base, int B, int N, int H, int d, int rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)H * d, (cuuint64_t)N * H * d};
    cuuint32_t box[4] = {128, 1, (cuuint32_t)rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bytes (fp8) [BH, nKB, d] centroids; box = 128 channels x 64 centroids x 1.
bool make_map_u8_cent(CUtensorMap *m, const void *base, int BH, int nKB, int d)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nKB, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)nKB * d};
    cuuint32_t box[3] = {128, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [BH, nKB, d] centroids; box = 64 channels x 64 centroids x 1.
bool make_map_cent(CUtensorMap *m, const void *base, int BH, int nKB, int d)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nKB, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)nKB * d * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 rows of a 2-D array [rows, d] with a row pitch; box = 64 channels x 1 row
// (the shape tile::gather4 takes).
bool make_map_rows(CUtensorMap *m, const void *base, int64_t rows, int d, int64_t pitch)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)pitch * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 cubes of the latent grid that follows a prefix of P tokens (B = 1):
// [T, Hs, Ws, H, d] seen through the token strides; box = 64 channels x 1 head
// x cW x cH x cT tokens, i.e. one cube's 64 token rows of 128 bytes, t-major.
bool make_map_cube(CUtensorMap *m, const void *base, int P, int H, int d, int gT, int gH, int gW, int cT, int cH,
                   int cW, int64_t sn, int64_t sh)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const __nv_bfloat16 *g0 = static_cast<const __nv_bfloat16 *>(base) + (int64_t)P * sn;
    cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)gW, (cuuint64_t)gH, (cuuint64_t)gT};
    cuuint64_t strides[4] = {(cuuint64_t)sh * 2, (cuuint64_t)sn * 2, (cuuint64_t)gW * sn * 2,
                             (cuuint64_t)gH * gW * sn * 2};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)cW, (cuuint32_t)cH, (cuuint32_t)cT};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<__nv_bfloat16 *>(g0), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool QK8, bool PV8>
cudaError_t launch_attn_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                               const CUtensorMap &tkc, const CUtensorMap &tvc, const CUtensorMap (&tg)[4],
                               const CUtensorMap (&t5)[3], const AttnArgs &a, int64_t items, cudaStream_t st)
{
    const size_t smem = Lay<D, QK8, PV8>::bytes(a.nW);
    cudaError_t e =
        cudaFuncSetAttribute(attn_kernel<D, QK8, PV8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    attn_kernel<D, QK8, PV8><<<(unsigned)items, kThreads, smem, st>>>(tq, tk, tv, tkc, tvc, tg[0], tg[1], tg[2],
                                                                      tg[3], t5[0], t5[1], t5[2], a);
    return cudaGetLastError();
}

}  // namespace

#ifdef BSA_TRACE
long long *g_trace = nullptr;
int g_trace_base = 0;
extern "C" __attribute__((visibility("default"))) void bsa_debug_set_trace(void *p, int base)
{
    g_trace = static_cast<long long *>(p);
    g_trace_base = base;
}
#endif

// Key-chunk split of the dense rows: enough items to cover the GPU, chunks of
// at least 256 key blocks, bounded by `max_partials` partial tiles.
int dense_split_for(const Dims &D, int nrows, int64_t max_partials)
{
    if (nrows <= 0) return 1;
    const int64_t tiles = (int64_t)D.B * D.H * ceil_div(nrows, kM);
    const int64_t fill = 2 * (int64_t)sm_count();
    if (tiles >= fill) return 1;
    int split = (int)std::min<int64_t>(ceil_div(D.nKB, 256), ceil_div(fill, tiles));
    split = std::max(1, split);
    while (split > 1 && tiles * split > max_partials) --split;
    return split;
}

int64_t dense_partial_tiles(const Dims &D, int nrows)
{
    const int split = dense_split_for(D, nrows, INT64_MAX);
    return split > 1 ? (int64_t)D.B * D.H * ceil_div(nrows, kM) * split : 0;
}

cudaError_t launch_attention(const bsa_params &p, const Dims &D, const void *q, const void *k,
                             const void *v, const float *kbar, const float *vbar,
                             const int64_t *row_ptr, const int32_t *col_idx, const int32_t *extra_idx,
                             const int32_t *extra_count, void *out, float *lse, int dense_only,
                             int row_begin, int row_end, char *ws, const WsLayout &L, cudaStream_t st,
                             int phase)
{
    // phase: 0 = everything, 1 = only the preparation kernels (bf16 copies,
    // centroids, modified centroids, gather lists), 2 = only the fine pass
    // (and the dense-row merge), which reads what phase 1 wrote.
    const bool prep = phase != 2, run = phase != 1;
    const int BH = D.B * D.H;
    int64_t sb = p.stride_b, sn = p.stride_n, sh = p.stride_h;
    const void *q16 = q, *k16 = k, *v16 = v;
    if (p.dtype == BSA_DT_F32) {
        // the tensor cores take bf16 operands: round the f32 inputs once
        const int64_t n = (int64_t)D.B * D.N * D.H * D.d;
        const unsigned g = (unsigned)std::min<int64_t>(ceil_div(n, 256), (int64_t)sm_count() * 16);
        __nv_bfloat16 *dq = reinterpret_cast<__nv_bfloat16 *>(ws + L.q16);
        __nv_bfloat16 *dk = reinterpret_cast<__nv_bfloat16 *>(ws + L.k16);
        __nv_bfloat16 *dv = reinterpret_cast<__nv_bfloat16 *>(ws + L.v16);
        if (prep) {
            count_launch();
            inputs_to_bf16_kernel<<<g, 256, 0, st>>>(static_cast<const float *>(q), dq, D.B, D.N, D.H, D.d, sb, sn, sh);
            count_launch();
            inputs_to_bf16_kernel<<<g, 256, 0, st>>>(static_cast<const float *>(k), dk, D.B, D.N, D.H, D.d, sb, sn, sh);
            count_launch();
            inputs_to_bf16_kernel<<<g, 256, 0, st>>>(static_cast<const float *>(v), dv, D.B, D.N, D.H, D.d, sb, sn, sh);
        }
        q16 = dq;
        k16 = dk;
        v16 = dv;
        sh = D.d;
        sn = (int64_t)D.H * D.d;
        sb = (int64_t)D.N * D.H * D.d;
    }
    __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(ws + L.kc16);
    __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(ws + L.vc16);
    const bool use_cent = !dense_only && p.centroid;
    if (use_cent && prep) {
        const int64_t n = (int64_t)BH * D.nKB * D.d;
        const unsigned g = (unsigned)std::min<int64_t>(ceil_div(n, 256), (int64_t)sm_count() * 8);
        count_launch();
        to_bf16_kernel<<<g, 256, 0, st>>>(kbar, kc, n);
        count_launch();
        to_bf16_kernel<<<g, 256, 0, st>>>(vbar, vc, n);
    }
    const bool f8 = p.qk_fp8 != 0;
    uint8_t *q8 = reinterpret_cast<uint8_t *>(ws + L.q8), *k8 = reinterpret_cast<uint8_t *>(ws + L.k8);
    uint8_t *kc8 = reinterpret_cast<uint8_t *>(ws + L.kc8);
    float *sq8 = reinterpret_cast<float *>(ws + L.sq8), *sk8 = reinterpret_cast<float *>(ws + L.sk8);
    float *skc8 = reinterpret_cast<float *>(ws + L.skc8);
    const int nb64 = (int)ceil_div(D.N, 64), nch64 = (int)ceil_div(D.nKB, 64);
    if (f8 && prep) {
        // Q per 64 tokens, K per key block (also 64 tokens), centroids per 64
        count_launch();
        quant_rows_kernel<<<dim3((unsigned)nb64, (unsigned)BH), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(q16), sb, sn, sh, D.N, D.H, nb64, q8, sq8);
        count_launch();
        quant_rows_kernel<<<dim3((unsigned)nb64, (unsigned)BH), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(k16), sb, sn, sh, D.N, D.H, nb64, k8, sk8);
        if (use_cent) count_launch();
        if (use_cent)
            quant_cent_kernel<<<dim3((unsigned)nch64, (unsigned)BH), 256, 0, st>>>(kbar, D.nKB, nch64, kc8, skc8);
    }
    const bool v8 = f8 && p.pv_fp8 != 0;
    uint8_t *v8p = reinterpret_cast<uint8_t *>(ws + L.v8), *vc8 = reinterpret_cast<uint8_t *>(ws + L.vc8);
    float *sv8 = reinterpret_cast<float *>(ws + L.sv8);
    if (v8 && prep) {
        // V and the value centroids with one scale per (b, h, channel)
        cudaError_t e = cudaMemsetAsync(sv8, 0, (size_t)BH * D.d * 4, st);
        if (e != cudaSuccess) return e;
        count_launch();
        vmax_kernel<<<dim3((unsigned)ceil_div(D.N, 256), (unsigned)BH), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(v16), sb, sn, sh, D.N, D.H, reinterpret_cast<uint32_t *>(sv8));
        count_launch();
        sv_scale_kernel<<<(unsigned)ceil_div(BH * D.d, 256), 256, 0, st>>>(reinterpret_cast<uint32_t *>(sv8),
                                                                             BH * D.d);
        count_launch();
        quant_v_kernel<<<dim3((unsigned)nb64, (unsigned)BH), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(v16), sb, sn, sh, D.N, D.H, sv8, v8p);
        if (use_cent) count_launch();
        if (use_cent)
            quant_vcent_kernel<<<dim3((unsigned)nch64, (unsigned)BH), 256, 0, st>>>(vbar, D.nKB, sv8, vc8);
    }
    CUtensorMap tq, tk, tv, tkc, tvc;
    if (f8) {
        const bool vm = v8 ? make_map_u8_bnhd(&tv, v8p, D.B, D.N, D.H, D.d, kBK) && make_map_u8_cent(&tvc, vc8, BH, D.nKB, D.d)
                           : make_map_bnhd(&tv, v16, D.B, D.N, D.H, D.d, sb, sn, sh, kBK) &&
                                 make_map_cent(&tvc, vc, BH, D.nKB, D.d);
        if (!make_map_u8_bnhd(&tq, q8, D.B, D.N, D.H, D.d, kM) || !make_map_u8_bnhd(&tk, k8, D.B, D.N, D.H, D.d, kBK) ||
            !vm || !make_map_u8_cent(&tkc, kc8, BH, D.nKB, D.d)) {
            set_error("cuTensorMapEncodeTiled failed for the fp8 tiles");
            return cudaErrorInvalidValue;
        }
    } else if (!make_map_bnhd(&tq, q16, D.B, D.N, D.H, D.d, sb, sn, sh, D.cube ? kBK : kM) ||
        !make_map_bnhd(&tk, k16, D.B, D.N, D.H, D.d, sb, sn, sh, kBK) ||
        !make_map_bnhd(&tv, v16, D.B, D.N, D.H, D.d, sb, sn, sh, kBK) ||
        !make_map_cent(&tkc, kc, BH, D.nKB, D.d) || !make_map_cent(&tvc, vc, BH, D.nKB, D.d)) {
        set_error("cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)");
        return cudaErrorInvalidValue;
    }
    CUtensorMap t5[3] = {tq, tk, tv};   // cube maps (unused without cube tiling)
    if (D.cube) {
        const int P = p.prefix_len;
        if (!make_map_cube(&t5[0], q16, P, D.H, D.d, p.grid_t, p.grid_h, p.grid_w, p.cube_t, p.cube_h, p.cube_w, sn,
                           sh) ||
            !make_map_cube(&t5[1], k16, P, D.H, D.d, p.grid_t, p.grid_h, p.grid_w, p.cube_t, p.cube_h, p.cube_w, sn,
                           sh) ||
            !make_map_cube(&t5[2], v16, P, D.H, D.d, p.grid_t, p.grid_h, p.grid_w, p.cube_t, p.cube_h, p.cube_w, sn,
                           sh)) {
            set_error("cuTensorMapEncodeTiled failed for the cube tiles");
            return cudaErrorInvalidValue;
        }
    }
    AttnArgs a;
    a.sq8 = sq8;
    a.sk8 = sk8;
    a.skc8 = skc8;
    a.nb64 = nb64;
    a.nch64 = nch64;
    a.sv8 = sv8;
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
    a.B = D.B;
    a.H = D.H;
    a.N = D.N;
    a.nQB = D.nQB;
    a.nKB = D.nKB;
    a.nW = D.nW;
    a.Bq = D.Bq;
    a.sb = p.stride_b;
    a.sn = p.stride_n;
    a.sh = p.stride_h;
    a.row_ptr = row_ptr;
    a.col_idx = col_idx;
    a.out = out;
    a.lse = lse;
    a.out_f32 = p.dtype == BSA_DT_F32;
    a.centroid = p.centroid;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D.d));
    a.status = reinterpret_cast<int32_t *>(ws + L.status);
#ifdef BSA_TRACE
    a.trace = g_trace;
    a.trace_base = g_trace_base;
#else
    a.trace = nullptr;
    a.trace_base = 0;
#endif
    a.E = dense_only ? 0 : D.E;
    a.Ecap = D.E > 0 ? std::min(D.E, D.nKB) : 0;
    a.extra_idx = extra_idx;
    a.extra_count = extra_count;
    a.kx = static_cast<const __nv_bfloat16 *>(k16);
    a.vx = static_cast<const __nv_bfloat16 *>(v16);
    a.xk16 = reinterpret_cast<const __nv_bfloat16 *>(ws + L.xk16);
    a.xv16 = reinterpret_cast<const __nv_bfloat16 *>(ws + L.xv16);
    a.xbias = reinterpret_cast<const float *>(ws + L.xbias);
    a.xcnt = reinterpret_cast<const int32_t *>(ws + L.xcnt);
    a.xoff = reinterpret_cast<const int64_t *>(ws + L.xoff);
    a.slot = reinterpret_cast<const int32_t *>(ws + L.mc_slot);
    if (a.E > 0 && p.dtype != BSA_DT_BF16) {
        // the gathers read rows through the input strides
        set_error("extra tokens need bf16 inputs");
        return cudaErrorInvalidValue;
    }
    if (a.E > 0 && prep) {
        McArgs m;
        m.extra_idx = extra_idx;
        m.extra_count = extra_count;
        m.rows = D.rows;
        m.H = D.H;
        m.N = D.N;
        m.nQB = D.nQB;
        m.nKB = D.nKB;
        m.E = D.E;
        m.G = mc_groups(D);
        m.rpg = (int)ceil_div(D.nQB, m.G);
        m.xcnt = reinterpret_cast<int32_t *>(ws + L.xcnt);
        m.xoff = reinterpret_cast<const int64_t *>(ws + L.xoff);
        m.cnt3 = reinterpret_cast<int32_t *>(ws + L.mc_cnt3);
        m.off3 = reinterpret_cast<const int64_t *>(ws + L.mc_off3);
        m.ent = reinterpret_cast<uint64_t *>(ws + L.mc_ent);
        m.slot = reinterpret_cast<int32_t *>(ws + L.mc_slot);
        m.xbias = reinterpret_cast<float *>(ws + L.xbias);
        m.cap = L.mc_cap;
        m.status = a.status;
        const int64_t n3 = BH * D.nKB * m.G;
        int64_t *tile = reinterpret_cast<int64_t *>(ws + L.mc_tile);
        const size_t gsm = (size_t)D.nKB * 4;
        cudaError_t e;
        if ((e = cudaFuncSetAttribute(mc_group_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsm)) !=
                cudaSuccess ||
            (e = cudaFuncSetAttribute(mc_group_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsm)) !=
                cudaSuccess)
            return e;
        count_launch();
        mc_count_kernel<<<(unsigned)ceil_div(D.rows, 8), 256, 0, st>>>(m);
        if ((e = launch_scan(m.xcnt, D.rows, reinterpret_cast<int64_t *>(ws + L.xoff), tile, st)) != cudaSuccess)
            return e;
        count_launch();
        mc_group_kernel<1><<<(unsigned)(BH * m.G), 256, gsm, st>>>(m);
        if ((e = launch_scan(m.cnt3, n3, reinterpret_cast<int64_t *>(ws + L.mc_off3), tile, st)) != cudaSuccess)
            return e;
        count_launch();
        mc_group_kernel<2><<<(unsigned)(BH * m.G), 256, gsm, st>>>(m);
        count_launch();
        if (D.d == 128)
            mc_build_kernel<128><<<(unsigned)(BH * D.nKB), 256, 0, st>>>(
                m, kbar, vbar, static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), sb, sn,
                sh, reinterpret_cast<__nv_bfloat16 *>(ws + L.xk16), reinterpret_cast<__nv_bfloat16 *>(ws + L.xv16));
        else
            mc_build_kernel<64><<<(unsigned)(BH * D.nKB), 128, 0, st>>>(
                m, kbar, vbar, static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), sb, sn,
                sh, reinterpret_cast<__nv_bfloat16 *>(ws + L.xk16), reinterpret_cast<__nv_bfloat16 *>(ws + L.xv16));
        const int64_t ntiles = (int64_t)BH * ceil_div(D.N, kM);
        count_launch();
        glist_kernel<<<(unsigned)ceil_div(ntiles, 4), 128, 0, st>>>(
            extra_idx, extra_count, D.E, D.nQB, D.Bq, (int)ceil_div(D.N, kM), ntiles,
            reinterpret_cast<uint32_t *>(ws + L.glist), reinterpret_cast<int32_t *>(ws + L.glcnt));
    }
    a.glist = reinterpret_cast<const uint32_t *>(ws + L.glist);
    a.glcnt = reinterpret_cast<const int32_t *>(ws + L.glcnt);
    a.n_sparse = dense_only ? 0 : (int)ceil_div(D.N, kM);
    a.skip_begin = row_begin;
    a.skip_end = row_end;
    const int nrows = std::max(0, row_end - row_begin);
    a.dense_begin = row_begin;
    a.dense_end = row_end;
    a.n_dense = (int)ceil_div(nrows, kM);
    a.dense_split = dense_split_for(D, nrows, L.part_tiles);
    a.split_blocks = (int)ceil_div(D.nKB, a.dense_split);
    a.part_o = reinterpret_cast<float *>(ws + L.part_o);
    a.part_ml = reinterpret_cast<float *>(ws + L.part_ml);
    const int64_t items = (int64_t)BH * (a.n_dense * (int64_t)a.dense_split + a.n_sparse);
    if (items == 0 || !run) return cudaGetLastError();
    // gather maps: token rows of K and V as one 2-D array when the strides allow it
    // (the row pitch min(sn, sh) divides every stride and holds a whole row), and the
    // modified centroids [mc_cap, d]
    CUtensorMap tg[4] = {tk, tv, tk, tv};
    a.gather_tma = 0;
    a.grow_b = a.grow_n = a.grow_h = 0;
    if (a.E > 0) {
        const int64_t rs = std::min(sn, sh);
        if (rs >= D.d && sb % rs == 0 && sn % rs == 0 && sh % rs == 0) {
            const int64_t nrows_k = (int64_t)(D.B - 1) * (sb / rs) + (int64_t)(D.N - 1) * (sn / rs) +
                                    (int64_t)(D.H - 1) * (sh / rs) + 1;
            const int64_t nrows_x = L.mc_cap;
            if (nrows_k < INT32_MAX && nrows_x < INT32_MAX && make_map_rows(&tg[0], k16, nrows_k, D.d, rs) &&
                make_map_rows(&tg[1], v16, nrows_k, D.d, rs) &&
                make_map_rows(&tg[2], ws + L.xk16, nrows_x, D.d, D.d) &&
                make_map_rows(&tg[3], ws + L.xv16, nrows_x, D.d, D.d)) {
                a.gather_tma = 1;
                a.grow_b = sb / rs;
                a.grow_n = sn / rs;
                a.grow_h = sh / rs;
            } else {
                tg[0] = tk;
                tg[1] = tv;
                tg[2] = tk;
                tg[3] = tv;
            }
        }
    }
    cudaError_t e = D.d == 64   ? launch_attn_kernel<64, false, false>(tq, tk, tv, tkc, tvc, tg, t5, a, items, st)
                    : v8        ? launch_attn_kernel<128, true, true>(tq, tk, tv, tkc, tvc, tg, t5, a, items, st)
                    : p.qk_fp8  ? launch_attn_kernel<128, true, false>(tq, tk, tv, tkc, tvc, tg, t5, a, items, st)
                                : launch_attn_kernel<128, false, false>(tq, tk, tv, tkc, tvc, tg, t5, a, items, st);
    if (e != cudaSuccess) return e;
    if (a.n_dense > 0 && a.dense_split > 1) {
        count_launch();
        combine_kernel<<<(unsigned)(BH * (int64_t)a.n_dense), kM, 0, st>>>(a, D.d);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace bsa
