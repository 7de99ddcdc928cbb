// lq_chunk.cu -- chunked prefill on the 5th-generation tensor cores (sm_100a):
// the FP32 recurrence of equation 1 ("LeapQuant: Efficient Linear Attention
// with Accurate Recurrent State Quantization", Appendix Table 4) over chunks
// of C = 64 tokens, for the scalar gate (Gated DeltaNet) with BF16 inputs and
// d_k = 128.  The prefill carries the FP32 state; snapshots for the prefix
// cache (Figure 1(b)) are quantized copies taken between passes.
//
// Within a chunk, from the state S_0 at its start (S in R^{d_v x d_k}), with
// L_t = sum_{s<=t} log alpha_s (t = 0..63, from the chunk start),
// G_tm = e^{L_t - L_m} and b_t = alpha_t k_t (or 0 when delta = 0):
//
//   A   = strictly lower (G .* beta_m (K K^T))    (0 when delta = 0)
//   P   = lower, with diagonal, (G .* beta_m (Q K^T))
//   T   = (I + A)^{-1},   PT = P T
//   R   = V - Diag(e^L) K S_0^T                   (V when delta = 0)
//   [O_intra; U] = [PT; T] R                      (U: the updates u_t)
//   O   = Diag(e^L) Q S_0^T + O_intra
//   S_C = e^{L_C} S_0 + (Diag(beta e^{L_C - L}) U)^T K
//
// which is the token recurrence u_t = v_t - S_{t-1} b_t, o_t = S_t q_t,
// S_t = alpha_t S_{t-1} + u_t (beta_t k_t)^T unrolled over the chunk.
//
// Two kernels per pass of up to kMaxPassChunks chunks:
//  * chunk_prep_kernel (every chunk of every head in parallel): K K^T and
//    Q K^T with warp-level tensor-core MMAs (BF16, exact products, FP32
//    sums; several CTAs share an SM), A and P on CUDA cores, then T and PT
//    column by column (forward substitution, FP32),
//    written to the caller's workspace as [PT; T] (128 x 64, three BF16 parts
//    of each FP32 value, in the operand layout: 48 KB per chunk and head);
//  * chunk_scan_kernel (one CTA per head and 64 value rows, the chunks of the
//    pass in order): the three products that carry the state, FP32-faithful
//    on the tensor core --
//      X   = [Q; K] S_0^T : BF16 x (S split into three BF16 parts)
//      [O_intra; U] = [PT; T] R : (three BF16 parts) x (three BF16 parts), the
//                         six cross products of parts p + q <= 2
//      D_S = K^T U^ : BF16 x (U^ = beta e^{L_C - L} U split into three BF16 parts)
//    with the state slice in registers of four epilogue warps between chunks.
// Every mbarrier wait is bounded (lq_common.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstddef>
#include <cstring>

#include "lq_kernels.h"
#include "lq_tc.cuh"

namespace lq {
namespace {

constexpr int kC = 64;           // tokens per chunk
constexpr int kDK = 128;         // key channels (the tensor-core path's d_k)
constexpr int kDVS = 64;         // value rows per scan CTA
constexpr int kQKBytes = 2 * kC * kDK * 2;   // [Q; K] BF16 operand: 32 KB
constexpr int kVBytes = kC * kDVS * 2;       // V slice: 8 KB
constexpr int kTRows = 2 * kC;               // [PT; T]
// [PT; T] of one chunk and head in the workspace: three BF16 parts of the
// K-major operand (element (r, m) of part p at byte p * 16384 +
// (m / 8) * 2048 + 16 r + 2 (m % 8)), 48 KB
constexpr int kTPartBytes = kTRows * kC * 2;
constexpr int kWsChunkBytes = 3 * kTPartBytes;

// ---------------------------------------------------------------------------
// TMA (tiled bulk tensor copies, no multicast)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// The [Q; K] operand of one chunk: K-major, no swizzle, 128 rows (rows 0..63
// the chunk's q_t, rows 64..127 its k_t) by d_k = 128 BF16 columns; element
// (row, j) at byte (j / 8) * 2048 + 16 row + 2 (j % 8).  Sixteen 8-column
// slabs of the two tensors, one TMA box {8 channels, 1 head, 64 tokens} each.
__device__ __forceinline__ void load_qk(unsigned char *qk, const CUtensorMap *qmap,
                                        const CUtensorMap *kmap, int h, int tok0, uint64_t *bar) {
#pragma unroll 1
    for (int s = 0; s < kDK / 8; ++s) {
        tma_load_3d(qk + s * 2048, qmap, 8 * s, h, tok0, bar);
        tma_load_3d(qk + s * 2048 + 1024, kmap, 8 * s, h, tok0, bar);
    }
}

// Two values in three BF16 parts each, packed in pairs (x0 in the low half).
__device__ __forceinline__ void split2_bf16x3(float x0, float x1, uint32_t &w0, uint32_t &w1,
                                              uint32_t &w2) {
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(x0, x1);
    const float2 b0 = __bfloat1622float2(p0);
    const float r0 = x0 - b0.x, r1 = x1 - b0.y;
    const __nv_bfloat162 p1 = __floats2bfloat162_rn(r0, r1);
    const float2 b1 = __bfloat1622float2(p1);
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(r0 - b1.x, r1 - b1.y);
    w0 = *reinterpret_cast<const uint32_t *>(&p0);
    w1 = *reinterpret_cast<const uint32_t *>(&p1);
    w2 = *reinterpret_cast<const uint32_t *>(&p2);
}

// The running log gate of a chunk, every lane: lane l holds L at tokens 2l
// and 2l+1 (inclusive sums of log alpha from the chunk start).
__device__ __forceinline__ void chunk_log_gate(const float *alpha_s, int lane, float &Le, float &Lo) {
    const float a0 = logf(alpha_s[2 * lane]), a1 = logf(alpha_s[2 * lane + 1]);
    float incl = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    Lo = incl;
    Le = incl - a1;
}

// L_t for token t (0..63) from the lane pairs of chunk_log_gate.
__device__ __forceinline__ float log_gate_at(float Le, float Lo, int t) {
    const float e = __shfl_sync(0xffffffffu, Le, t >> 1);
    const float o = __shfl_sync(0xffffffffu, Lo, t >> 1);
    return (t & 1) ? o : e;
}

// ---------------------------------------------------------------------------
// Phase 1: [PT; T] of every chunk of the pass
// ---------------------------------------------------------------------------

constexpr int kPrepThreads = 128;
constexpr int kAStride = 68;  // padded row stride (floats) of A, P and the solved columns

struct PrepSmem {
    alignas(16) float A[kC][kAStride];  // strictly lower (G .* beta_m K K^T)
    alignas(16) float P[kC][kAStride];  // lower (G .* beta_m Q K^T)
    alignas(16) float L2[kC];           // L_t log2(e)
    alignas(16) float beta[kC];
    float alpha[kC];
    uint64_t bar_in;
};

// Four 8 x 8 BF16 matrices of the [Q; K] tile into the fragment registers of
// a warp-level MMA; lane i addresses row i % 8 of matrix i / 8.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const unsigned char *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

// D += A B for one 16 x 8 tile, K = 16: BF16 inputs, FP32 accumulation.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__host__ __device__ constexpr int prep_smem_bytes() {
    return kQKBytes + (int)sizeof(PrepSmem) + 128;
}

// Column m of T = (I + A)^{-1}: forward substitution in blocks of 8 rows, the
// block's rows accumulated together against the solved rows above it (read
// back from X[m], the column's row of the solved-column store).  Two lanes
// (xor 1) share a column: each sums every other group of 4 solved rows, one
// shuffle joins the halves, and both finish the block's own 8 x 8 triangle.
__device__ __forceinline__ void solve_column(const PrepSmem &ps, float *Xm, int m, int half) {
#pragma unroll 1
    for (int blk = 0; blk < kC / 8; ++blk) {
        const int r0 = 8 * blk;
        float acc[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] = 0.0f;
#pragma unroll 1
        for (int n = 4 * half; n < r0; n += 8) {
            const float4 xv = *reinterpret_cast<const float4 *>(Xm + n);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float4 av = *reinterpret_cast<const float4 *>(&ps.A[r0 + r][n]);
                acc[r] = fmaf(av.x, xv.x, acc[r]);
                acc[r] = fmaf(av.y, xv.y, acc[r]);
                acc[r] = fmaf(av.z, xv.z, acc[r]);
                acc[r] = fmaf(av.w, xv.w, acc[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
        float xb[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float v = (r0 + r == m ? 1.0f : 0.0f) - acc[r];
#pragma unroll
            for (int n = 0; n < r; ++n) v = fmaf(-ps.A[r0 + r][r0 + n], xb[n], v);
            xb[r] = v;
        }
        if (half == 0) {
            *reinterpret_cast<float4 *>(Xm + r0) = make_float4(xb[0], xb[1], xb[2], xb[3]);
            *reinterpret_cast<float4 *>(Xm + r0 + 4) = make_float4(xb[4], xb[5], xb[6], xb[7]);
        }
        __syncwarp();
    }
}

__global__ void __launch_bounds__(kPrepThreads) chunk_prep_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const ChunkArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *qk = smem;
    PrepSmem &ps = *reinterpret_cast<PrepSmem *>(smem + kQKBytes);
    // after the MMA the [Q; K] tile is dead: its space holds the solved
    // columns, X[m][t] = T[t][m] (row stride kAStride)
    float *X = reinterpret_cast<float *>(qk);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x % a.nc, bh = blockIdx.x / a.nc;
    const int b = bh / a.H, h = bh % a.H;
    const int tok0 = b * a.T_total + a.t0 + c * kC;  // flattened (sequence, token) row

    if (tid == 0) mbar_init(&ps.bar_in, 1);
    // gates of the chunk
    if (tid < kC) ps.alpha[tid] = a.alpha[((size_t)tok0 + tid) * a.H + h];
    else ps.beta[tid - kC] = a.beta[((size_t)tok0 + tid - kC) * a.H + h];
    __syncthreads();

    if (tid == 0) {
        mbar_arrive_expect_tx(&ps.bar_in, kQKBytes);
        load_qk(qk, &qmap, &kmap, h, tok0, &ps.bar_in);
    }
    if (warp == 1) {
        // L_t log2(e) of the chunk
        float Le, Lo;
        chunk_log_gate(ps.alpha, lane, Le, Lo);
        ps.L2[2 * lane] = Le * 1.4426950408889634f;
        ps.L2[2 * lane + 1] = Lo * 1.4426950408889634f;
    }
    // every thread observes the copies' completion (the tile is read through
    // the generic proxy), and L is in shared memory after the barrier
    const bool ok = mbar_wait_bounded(&ps.bar_in, 0);
    const bool good = !named_sync_or<1, kPrepThreads>(!ok);
    if (good) {
        // D[128 x 64] = [Q; K] K^T with warp-level MMAs (exact BF16 products,
        // FP32 sums): warp w takes rows 32w..32w+31 -- Q K^T for warps 0-1,
        // K K^T for warps 2-3 -- as two 16-row tiles by eight 8-column tiles.
        // (A tcgen05 product here would hold the kernel to one CTA per SM;
        // its time is the CUDA-core phases below, which want several.)
        float d[2][8][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) d[mt][nt][e] = 0.0f;
        const int mi = lane >> 3, ri = lane & 7;  // this lane's matrix and row in ldmatrix
#pragma unroll 2
        for (int k16 = 0; k16 < kDK / 16; ++k16) {
            // A tiles: matrices (rows +0 / +8) x (channels +0 / +8)
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int row = 32 * warp + 16 * mt + 8 * (mi & 1) + ri;
                ldmatrix_x4(af[mt], qk + (2 * k16 + (mi >> 1)) * 2048 + 16 * row);
            }
            // B = K^T: token n's row of K, channels +0 / +8, two 8-token tiles
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bf[4];
                const int n = 16 * np + 8 * (mi >> 1) + ri;
                ldmatrix_x4(bf, qk + (2 * k16 + (mi & 1)) * 2048 + 1024 + 16 * n);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    mma_bf16_16816(d[mt][2 * np], af[mt], bf[0], bf[1]);
                    mma_bf16_16816(d[mt][2 * np + 1], af[mt], bf[2], bf[3]);
                }
            }
        }
        // element (row, m) of the product: P (rows 0..63) or A (rows
        // 64..127) with the gate ratio e^{L_t - L_m} = 2^{(L_t - L_m) log2 e}
        // and beta_m; a thread holds rows g, g + 8 of each 16-row tile and
        // columns 2c, 2c + 1 of each 8-column tile
        const int g = lane >> 2, c2 = 2 * (lane & 3);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 32 * warp + 16 * mt + 8 * hr + g, t = r & (kC - 1);
                const bool qrow = r < kC;
                const float Lt = ps.L2[t];
                float *rowp = qrow ? ps.P[t] : ps.A[t];
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const int m = 8 * nt + c2;
                    const float2 lm = *reinterpret_cast<const float2 *>(&ps.L2[m]);
                    const float2 bm = *reinterpret_cast<const float2 *>(&ps.beta[m]);
                    const bool k0 = qrow ? (m <= t) : (m < t && a.delta);
                    const bool k1 = qrow ? (m + 1 <= t) : (m + 1 < t && a.delta);
                    const float v0 = k0 ? bm.x * d[mt][nt][2 * hr] * exp2f(Lt - lm.x) : 0.0f;
                    const float v1 = k1 ? bm.y * d[mt][nt][2 * hr + 1] * exp2f(Lt - lm.y) : 0.0f;
                    *reinterpret_cast<float2 *>(rowp + m) = make_float2(v0, v1);
                }
            }
    }
    // every warp's reads of the [Q; K] tile are done before it holds X
    const bool bad = named_sync_or<1, kPrepThreads>(!good);
    if (bad) return;

    unsigned char *wsb = reinterpret_cast<unsigned char *>(a.ws) + ((size_t)c * a.B * a.H + bh) * kWsChunkBytes;
    // T, column by column (two threads per column), into X
    {
        const int m = tid >> 1;
        solve_column(ps, X + m * kAStride, m, tid & 1);
    }
    named_sync<1, kPrepThreads>();
    // PT = P T: column m, rows in blocks of 8; thread (m, half) takes the
    // blocks {0, 3, 4, 7} or {1, 2, 5, 6} (equal work: P is lower triangular)
    {
        const int m = tid & (kC - 1), half = tid >> 6;
        const float *Xm = X + m * kAStride;
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
            const int blk = half ? (k == 0 ? 1 : k == 1 ? 2 : k == 2 ? 5 : 6)
                                 : (k == 0 ? 0 : k == 1 ? 3 : k == 2 ? 4 : 7);
            const int r0 = 8 * blk;
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = 0.0f;
#pragma unroll 1
            for (int n = 0; n < r0 + 8; n += 4) {
                const float4 xv = *reinterpret_cast<const float4 *>(Xm + n);
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float4 pv = *reinterpret_cast<const float4 *>(&ps.P[r0 + r][n]);
                    acc[r] = fmaf(pv.x, xv.x, acc[r]);
                    acc[r] = fmaf(pv.y, xv.y, acc[r]);
                    acc[r] = fmaf(pv.z, xv.z, acc[r]);
                    acc[r] = fmaf(pv.w, xv.w, acc[r]);
                }
            }
            // PT rows into the (no longer needed) A buffer, row-major
#pragma unroll
            for (int r = 0; r < 8; ++r) ps.A[r0 + r][m] = acc[r];
        }
    }
    named_sync<1, kPrepThreads>();
    // row r of [PT; T] (PT row r, or T row r - 64 read down column X[.][r - 64])
    // as three BF16 parts in the operand layout; a warp writes 512 contiguous
    // bytes per 8-column group and part
    {
        const int r = tid;
        float x[kC];
        if (r < kC) {
#pragma unroll
            for (int m = 0; m < kC; ++m) x[m] = ps.A[r][m];
        } else {
#pragma unroll
            for (int m = 0; m < kC; ++m) x[m] = X[m * kAStride + (r - kC)];
        }
#pragma unroll
        for (int g = 0; g < kC / 8; ++g) {
            uint32_t p0[4], p1[4], p2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) split2_bf16x3(x[8 * g + 2 * e], x[8 * g + 2 * e + 1], p0[e], p1[e], p2[e]);
            unsigned char *d = wsb + g * 2048 + 16 * r;
            *reinterpret_cast<uint4 *>(d) = make_uint4(p0[0], p0[1], p0[2], p0[3]);
            *reinterpret_cast<uint4 *>(d + kTPartBytes) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
            *reinterpret_cast<uint4 *>(d + 2 * kTPartBytes) = make_uint4(p2[0], p2[1], p2[2], p2[3]);
        }
    }
}

// ---------------------------------------------------------------------------
// Phase 2: the chunks of the pass in order, the state carried on the tensor core
// ---------------------------------------------------------------------------

// 8 epilogue warps: warp w serves TMEM lane quarter w % 4 and the 32
// accumulator columns 32 (w / 4) .. 32 (w / 4) + 31 (value rows of the slice).
// Warp 8 issues the MMAs, warp 9 loads the chunk inputs, lane 0 of warp 10
// brings each chunk's [PT; T] operand in with bulk copies.
constexpr int kEpiWarps = 8, kMmaWarp = 8, kLoadWarp = 9, kTWarp = 10;
constexpr int kScanThreads = (kEpiWarps + 3) * 32;
constexpr int kHalf = kDVS / 2;  // accumulator columns per epilogue thread

// TMEM columns (256 allocated): the three accumulators
constexpr uint32_t kColX = 0, kColOU = 64, kColS = 128;

struct ScanBars {
    uint64_t full[2], empty[2];          // input stages (TMA + cp.async)
    uint64_t t_full, t_empty;            // [PT; T] operand in shared memory (bulk copies)
    uint64_t x_done, ou_done, s_done;    // MMA completions
    uint64_t r_ready, u_ready, s_ready;  // operands written by the epilogue
    uint32_t tmem;
};

struct ScanLayout {
    int bars, qk, v, ab, s3, ru, tt, bytes;
};

__host__ __device__ constexpr ScanLayout scan_layout() {
    ScanLayout L{};
    L.bars = 0;
    L.qk = 1024;                          // [2][32 KB]
    L.v = L.qk + 2 * kQKBytes;            // [2][8 KB] V slice, [64 t][64 i], 128-byte swizzle
                                          // (1024-byte aligned)
    L.ab = L.v + 2 * kVBytes;             // [2][alpha 64, beta 64]
    L.s3 = L.ab + 2 * 512;                // [3][16 KB] S^T split (MN-major B of the X product)
    L.ru = L.s3 + 3 * 16384;              // [3][8 KB] R, then U^ (MN-major B, BF16 parts)
    L.tt = L.ru + 3 * 8192;               // [3][16 KB] [PT; T] (K-major A, BF16 parts)
    L.bytes = L.tt + 3 * 16384;
    return L;
}

// Writes values x[8 g' .. 8 g' + 7] (g' = 0..N/8-1) as three BF16 parts: the
// 16-byte word of each part at dst + part * part_bytes + (g0 + g') * stride.
template <int N>
__device__ __forceinline__ void store_parts(unsigned char *dst, const float (&x)[N], float scale,
                                            int g0, int stride, int part_bytes) {
#pragma unroll
    for (int g = 0; g < N / 8; ++g) {
        uint32_t a[4], b[4], c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            split2_bf16x3(scale * x[8 * g + 2 * e], scale * x[8 * g + 2 * e + 1], a[e], b[e], c[e]);
        unsigned char *d = dst + (g0 + g) * stride;
        *reinterpret_cast<uint4 *>(d) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4 *>(d + part_bytes) = make_uint4(b[0], b[1], b[2], b[3]);
        *reinterpret_cast<uint4 *>(d + 2 * part_bytes) = make_uint4(c[0], c[1], c[2], c[3]);
    }
}

__global__ void __launch_bounds__(kScanThreads, 1) chunk_scan_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, const ChunkArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // the swizzled V tiles need 1024-byte aligned addresses: align the base
    // (the launch reserves 1 KB for it)
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    constexpr ScanLayout SL = scan_layout();
    ScanBars &sb = *reinterpret_cast<ScanBars *>(smem + SL.bars);
    unsigned char *qkbuf = smem + SL.qk;
    unsigned char *vbuf = smem + SL.v;
    float *abbuf = reinterpret_cast<float *>(smem + SL.ab);
    unsigned char *s3 = smem + SL.s3;
    unsigned char *ru = smem + SL.ru;
    unsigned char *tt = smem + SL.tt;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nsl = a.DV / kDVS;
    const int bh = blockIdx.x / nsl, i0 = (blockIdx.x % nsl) * kDVS;
    const int b = bh / a.H, h = bh % a.H;
    const int nc = a.nc;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sb.full[s], 33);  // 32 loader lanes' gate copies + the TMA arrival
            mbar_init(&sb.empty[s], kEpiWarps);
        }
        mbar_init(&sb.t_full, 1);
        mbar_init(&sb.t_empty, 1);
        mbar_init(&sb.x_done, 1);
        mbar_init(&sb.ou_done, 1);
        mbar_init(&sb.s_done, 1);
        mbar_init(&sb.r_ready, 4);
        mbar_init(&sb.u_ready, 4);
        mbar_init(&sb.s_ready, kEpiWarps);
    }
    if (warp == kMmaWarp) tmem_alloc(&sb.tmem, 256);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = sb.tmem;

    if (warp == kLoadWarp) {
        // ---------------------------------------------------------- loader
        int c = 0;
        for (; c < nc; ++c) {
            const int s = c & 1;
            if (c >= 2 && !mbar_wait_bounded(&sb.empty[s], ((c >> 1) - 1) & 1)) break;
            const int tok0 = b * a.T_total + a.t0 + c * kC;
            float *ab = abbuf + s * 128;
            // gates: lane l copies tokens l and l + 32 of alpha and beta
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int t = lane + 32 * u;
                cp_async4(ab + t, a.alpha + ((size_t)tok0 + t) * a.H + h);
                cp_async4(ab + kC + t, a.beta + ((size_t)tok0 + t) * a.H + h);
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&sb.full[s]))
                         : "memory");
            if (lane == 0) {
                mbar_arrive_expect_tx(&sb.full[s], kQKBytes + kVBytes);
                load_qk(qkbuf + s * kQKBytes, &qmap, &kmap, h, tok0, &sb.full[s]);
                tma_load_3d(vbuf + s * kVBytes, &vmap, i0, h, tok0, &sb.full[s]);
            }
        }
        // drain copies still in flight into this CTA (after an expired wait)
        for (int j = c - 1; j >= 0 && j >= c - 2; --j) mbar_wait_bounded(&sb.full[j & 1], (j >> 1) & 1);
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idx = idesc_bf16(128, kDVS, false, true);
            constexpr uint32_t ids = idesc_bf16(128, kDVS, true, true);
            // descriptors at offset 0; an operand offset of o bytes adds o >> 4
            const uint64_t dS = smem_desc(smem_u32(s3), 128, 2048);     // S^T parts (MN-major B)
            const uint64_t dT = smem_desc(smem_u32(tt), 2048, 128);     // [PT; T] parts (K-major A)
            const uint64_t dR = smem_desc(smem_u32(ru), 128, 1024);     // R / U^ parts (MN-major B)
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1, ph = c & 1;
                if (!mbar_wait_bounded(&sb.full[s], (c >> 1) & 1)) break;
                if (!mbar_wait_bounded(&sb.s_ready, ph)) break;
                tc_fence_after_sync();
                const uint64_t dQK = smem_desc(smem_u32(qkbuf + s * kQKBytes), 2048, 128);
                const uint64_t dKT = smem_desc(smem_u32(qkbuf + s * kQKBytes + 1024), 128, 2048);
                // X = [Q; K] S^T, S = s0 + s1 + s2 (smallest part first)
#pragma unroll
                for (int k16 = 0; k16 < kDK / 16; ++k16)
#pragma unroll
                    for (int p = 2; p >= 0; --p)
                        mma_bf16(tm + kColX, dQK + ((k16 * 4096) >> 4), dS + ((p * 16384 + k16 * 256) >> 4),
                                 idx, k16 > 0 || p < 2);
                mma_commit(&sb.x_done);
                if (!mbar_wait_bounded(&sb.r_ready, ph)) break;
                if (!mbar_wait_bounded(&sb.t_full, ph)) break;
                tc_fence_after_sync();
                // [O_intra; U] = [PT; T] R: parts (p, q) with p + q <= 2, smallest first
#pragma unroll
                for (int k16 = 0; k16 < kC / 16; ++k16)
#pragma unroll
                    for (int n = 0; n < 6; ++n) {
                        constexpr int kP[6] = {2, 1, 0, 1, 0, 0}, kQ[6] = {0, 1, 2, 0, 1, 0};
                        mma_bf16(tm + kColOU, dT + ((kP[n] * 16384 + k16 * 4096) >> 4),
                                 dR + ((kQ[n] * 8192 + k16 * 256) >> 4), idx, k16 > 0 || n > 0);
                    }
                mma_commit(&sb.ou_done);
                mma_commit(&sb.t_empty);
                if (!mbar_wait_bounded(&sb.u_ready, ph)) break;
                tc_fence_after_sync();
                // D_S = K^T U^, U^ = u0 + u1 + u2
#pragma unroll
                for (int k16 = 0; k16 < kC / 16; ++k16)
#pragma unroll
                    for (int p = 2; p >= 0; --p)
                        mma_bf16(tm + kColS, dKT + ((k16 * 256) >> 4), dR + ((p * 8192 + k16 * 256) >> 4), ids,
                                 k16 > 0 || p < 2);
                mma_commit(&sb.s_done);
            }
        }
    } else if (warp == kTWarp) {
        // ---------------------------------------------------------- [PT; T] operand
        // the chunk's three BF16 parts, already in the operand layout in the
        // workspace, by bulk copies once the previous chunk's MMAs read them
        if (lane == 0) {
            int c = 0;
            for (; c < nc; ++c) {
                if (c >= 1 && !mbar_wait_bounded(&sb.t_empty, (c - 1) & 1)) break;
                const unsigned char *src =
                    reinterpret_cast<const unsigned char *>(a.ws) + ((size_t)c * a.B * a.H + bh) * kWsChunkBytes;
                mbar_arrive_expect_tx(&sb.t_full, kWsChunkBytes);
                for (int p = 0; p < 3; ++p) bulk_g2s(tt + p * kTPartBytes, src + p * kTPartBytes, kTPartBytes, &sb.t_full);
            }
            if (c > 0) mbar_wait_bounded(&sb.t_full, (c - 1) & 1);  // drain (after an expired wait)
        }
    } else {
        // ---------------------------------------------------------- epilogue (warps 0..7)
        const int qtr = warp & 3, hf = warp >> 2;
        const int r = 32 * qtr + lane;     // TMEM lane (row of the accumulators)
        const int t = r & (kC - 1);        // token of this row (rows 0..63 Q / O, 64..127 K / U)
        const int c0 = hf * kHalf;         // this thread's accumulator columns c0 .. c0 + 31
        const uint32_t ta = tm + ((uint32_t)(32 * qtr) << 16) + c0;
        float S[kHalf];                    // S[i0 + c0 + i][j = r], i = 0..31
        {
            const float *Sg = a.S + ((size_t)bh * a.DV + i0 + c0) * kDK + r;
#pragma unroll
            for (int i = 0; i < kHalf; ++i) S[i] = Sg[(size_t)i * kDK];
        }
        // S^T (MN-major B: N = value row i, K = key channel j = r), three BF16 parts
        auto write_s3 = [&]() {
            store_parts(s3 + 16 * r, S, 1.0f, c0 / 8, 2048, 16384);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.s_ready);
        };
        write_s3();
        bool ok = true;
        for (int c = 0; c < nc && ok; ++c) {
            const int s = c & 1, ph = c & 1;
            if (!mbar_wait_bounded(&sb.full[s], (c >> 1) & 1)) { ok = false; break; }
            const float *al = abbuf + s * 128, *be = al + kC;
            float Le, Lo;
            chunk_log_gate(al, lane, Le, Lo);
            const float Lt = log_gate_at(Le, Lo, t);
            const float LC = __shfl_sync(0xffffffffu, Lo, 31);
            const float eLt = expf(Lt);
            if (!mbar_wait_bounded(&sb.x_done, ph)) { ok = false; break; }
            tc_fence_after_sync();
            if (r >= kC) {
                // R_t = v_t - e^{L_t} (S_0 k_t) (or v_t when delta = 0), three BF16 parts
                float xk[kHalf];
                tmem_load<32>(ta + kColX, xk);
                const unsigned char *vr = vbuf + s * kVBytes + t * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // the V tile is stored with the 128-byte swizzle: 16-byte
                    // chunk k of row t sits at chunk k ^ (t % 8), so the eight
                    // rows a quarter-warp reads hit distinct banks
                    const uint4 w = *reinterpret_cast<const uint4 *>(vr + 16 * ((c0 / 8 + q) ^ (t & 7)));
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float v = __uint_as_float((e & 1) ? (ww[e / 2] & 0xFFFF0000u) : (ww[e / 2] << 16));
                        xk[8 * q + e] = a.delta ? fmaf(-eLt, xk[8 * q + e], v) : v;
                    }
                }
                store_parts(ru + 16 * t, xk, 1.0f, c0 / 8, 1024, 8192);
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.r_ready);
            }
            if (!mbar_wait_bounded(&sb.ou_done, ph)) { ok = false; break; }
            tc_fence_after_sync();
            if (r < kC) {
                // o_t = e^{L_t} (S_0 q_t) + O_intra_t
                float xq[kHalf], oi[kHalf];
                tmem_load<32>(ta + kColX, xq);
                tmem_load<32>(ta + kColOU, oi);
                __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o) +
                                    (((size_t)b * a.T_total + a.t0 + c * kC + t) * a.H + h) * a.DV + i0 + c0;
#pragma unroll
                for (int q = 0; q < kHalf / 8; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 p = __floats2bfloat162_rn(fmaf(eLt, xq[8 * q + 2 * e], oi[8 * q + 2 * e]),
                                                                       fmaf(eLt, xq[8 * q + 2 * e + 1], oi[8 * q + 2 * e + 1]));
                        w[e] = *reinterpret_cast<const uint32_t *>(&p);
                    }
                    *reinterpret_cast<uint4 *>(og + 8 * q) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
                // U^_t = beta_t e^{L_C - L_t} u_t in three BF16 parts (MN-major B of K^T U^)
                float u[kHalf];
                tmem_load<32>(ta + kColOU, u);
                store_parts(ru + 16 * t, u, be[t] * expf(LC - Lt), c0 / 8, 1024, 8192);
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.u_ready);
            }
            if (!mbar_wait_bounded(&sb.s_done, ph)) { ok = false; break; }
            tc_fence_after_sync();
            {
                // S_C = e^{L_C} S_0 + (U^ ^T K)^T, column r of the slice
                float ds[kHalf];
                tmem_load<32>(ta + kColS, ds);
                const float eLC = expf(LC);
#pragma unroll
                for (int i = 0; i < kHalf; ++i) S[i] = fmaf(eLC, S[i], ds[i]);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.empty[s]);
            if (c + 1 < nc) write_s3();
        }
        if (ok) {
            float *Sg = a.S + ((size_t)bh * a.DV + i0 + c0) * kDK + r;
#pragma unroll
            for (int i = 0; i < kHalf; ++i) Sg[(size_t)i * kDK] = S[i];
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tm, 256);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// A 3-D map of a BF16 activation [B*T, H, D] (innermost D): box {box_d, 1, 64};
// swizzle128 stores each 128-byte box row with the 128-byte swizzle.
bool activation_map(CUtensorMap *m, const void *base, int D, int H, long long BT, int box_d,
                    bool swizzle128 = false) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)BT};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)box_d, 1, (cuuint32_t)kC};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t chunk_workspace_bytes(int BH, int chunks) {
    return (size_t)chunks * BH * kWsChunkBytes;
}

bool chunk_path_supported(int d_k, int d_v, int gate, bool bf16) {
    return bf16 && gate == 0 && d_k == kDK && (d_v == 64 || d_v == 128);
}

namespace {
// Sets the kernels' shared-memory limits once per device.
cudaError_t configure_chunk_kernels() {
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 prep_smem_bytes());
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(chunk_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     scan_layout().bytes + 1024);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    return cudaSuccess;
}
}  // namespace

cudaError_t launch_chunk_prep(const ChunkArgs &a, const void *q, const void *k, cudaStream_t stream) {
    if (a.nc < 1 || a.DV % kDVS != 0) return cudaErrorInvalidValue;
    cudaError_t e = configure_chunk_kernels();
    if (e != cudaSuccess) return e;
    const long long BT = (long long)a.B * a.T_total;
    CUtensorMap qm, km;
    if (!activation_map(&qm, q, kDK, a.H, BT, 8) || !activation_map(&km, k, kDK, a.H, BT, 8))
        return cudaErrorInvalidValue;
    chunk_prep_kernel<<<a.nc * a.B * a.H, kPrepThreads, prep_smem_bytes(), stream>>>(qm, km, a);
    return cudaGetLastError();
}

cudaError_t launch_chunk_scan(const ChunkArgs &a, const void *q, const void *k, const void *v,
                              cudaStream_t stream) {
    if (a.nc < 1 || a.DV % kDVS != 0) return cudaErrorInvalidValue;
    cudaError_t e = configure_chunk_kernels();
    if (e != cudaSuccess) return e;
    const long long BT = (long long)a.B * a.T_total;
    CUtensorMap qm, km, vm;
    if (!activation_map(&qm, q, kDK, a.H, BT, 8) || !activation_map(&km, k, kDK, a.H, BT, 8) ||
        !activation_map(&vm, v, a.DV, a.H, BT, kDVS, true))
        return cudaErrorInvalidValue;
    const int BH = a.B * a.H;
    chunk_scan_kernel<<<BH * (a.DV / kDVS), kScanThreads, scan_layout().bytes + 1024, stream>>>(qm, km, vm, a);
    return cudaGetLastError();
}

}  // namespace lq
