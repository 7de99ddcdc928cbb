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
//    Q K^T on the tensor core (BF16, exact products, FP32 sums), A and P on
//    CUDA cores, then T and PT column by column (forward substitution, FP32),
//    written to the caller's workspace as [PT; T] (128 x 64 FP32 per chunk);
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
constexpr int kWsChunkFloats = kTRows * kC;  // 8192 floats = 32 KB per chunk and head

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

// Descriptor of the K-major [Q; K] operand at K-step k16 (16 channels).
__device__ __forceinline__ uint64_t desc_qk(const unsigned char *qk, int k16) {
    return smem_desc(smem_u32(qk + k16 * 4096), 2048, 128);
}

// The chunk's K rows read as an MN-major operand K^T (M = key channel j,
// K = token t): element (j, t) at 1024 + (j / 8) * 2048 + (t / 8) * 128 +
// 16 (t % 8) + 2 (j % 8), i.e. LBO (K groups) = 128, SBO (MN groups) = 2048.
__device__ __forceinline__ uint64_t desc_kt_mn(const unsigned char *qk, int k16) {
    return smem_desc(smem_u32(qk + 1024 + k16 * 256), 128, 2048);
}

// Three BF16 parts with x = p0 + p1 + p2 + O(2^-24 |x|): each part is the
// nearest BF16 to the remainder (the remainders are exact FP32 differences).
__device__ __forceinline__ void split_bf16x3(float x, __nv_bfloat16 &p0, __nv_bfloat16 &p1,
                                             __nv_bfloat16 &p2) {
    p0 = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(p0);
    p1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(p1);
    p2 = __float2bfloat16_rn(r2);
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
constexpr int kAStride = 68;  // padded row stride (floats) of A and P in shared memory

struct PrepSmem {
    alignas(16) float A[kC][kAStride];
    alignas(16) float P[kC][kAStride];
    float alpha[kC], beta[kC];
    uint64_t bar_in, bar_mma;
    uint32_t tmem;
};

__host__ __device__ constexpr int prep_smem_bytes() {
    return kQKBytes + (int)sizeof(PrepSmem) + 128;
}

__global__ void __launch_bounds__(kPrepThreads) chunk_prep_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const ChunkArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *qk = smem;
    PrepSmem &ps = *reinterpret_cast<PrepSmem *>(smem + kQKBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x % a.nc, bh = blockIdx.x / a.nc;
    const int b = bh / a.H, h = bh % a.H;
    const int tok0 = b * a.T_total + a.t0 + c * kC;  // flattened (sequence, token) row

    if (tid == 0) {
        mbar_init(&ps.bar_in, 1);
        mbar_init(&ps.bar_mma, 1);
    }
    if (warp == 0) tmem_alloc(&ps.tmem, 64);
    // gates of the chunk
    if (tid < kC) ps.alpha[tid] = a.alpha[((size_t)tok0 + tid) * a.H + h];
    else ps.beta[tid - kC] = a.beta[((size_t)tok0 + tid - kC) * a.H + h];
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    bool ok = true;
    if (tid == 0) {
        mbar_arrive_expect_tx(&ps.bar_in, kQKBytes);
        load_qk(qk, &qmap, &kmap, h, tok0, &ps.bar_in);
        ok = mbar_wait_bounded(&ps.bar_in, 0);
        if (ok) {
            // D[128 x 64] = [Q; K] K^T: rows 0..63 Q K^T, rows 64..127 K K^T
            constexpr uint32_t idesc = idesc_bf16(128, kC, false, false);
#pragma unroll 1
            for (int k16 = 0; k16 < kDK / 16; ++k16) {
                const uint64_t bd = smem_desc(smem_u32(qk + 1024 + k16 * 4096), 2048, 128);
                mma_bf16(ps.tmem, desc_qk(qk, k16), bd, idesc, k16 > 0);
            }
            mma_commit(&ps.bar_mma);
        }
    }
    // every thread: L of the chunk (each warp computes it for itself)
    float Le, Lo;
    chunk_log_gate(ps.alpha, lane, Le, Lo);
    const int r = tid, t = r & (kC - 1);
    const bool qrow = r < kC;
    const float Lt = log_gate_at(Le, Lo, t);
    // thread 0's copies and MMAs went through, and the MMAs completed
    bool good = !named_sync_or<1, kPrepThreads>(tid == 0 && !ok);
    if (good) good = mbar_wait_bounded(&ps.bar_mma, 0);
    if (good) {
        tc_fence_after_sync();
        float x[64];
        const uint32_t ta = ps.tmem + ((uint32_t)(32 * warp) << 16);
        tmem_load<64>(ta, x);
        float *row = qrow ? ps.P[t] : ps.A[t];
#pragma unroll
        for (int m4 = 0; m4 < kC / 4; ++m4) {
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = 4 * m4 + e;
                const float Lm = log_gate_at(Le, Lo, m);
                const bool keep = qrow ? (m <= t) : (m < t && a.delta);
                v[e] = keep ? ps.beta[m] * x[m] * expf(Lt - Lm) : 0.0f;
            }
            *reinterpret_cast<float4 *>(row + 4 * m4) = make_float4(v[0], v[1], v[2], v[3]);
        }
    }
    tc_fence_before_sync();
    const bool bad = named_sync_or<1, kPrepThreads>(!good);
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(ps.tmem, 64);
    }
    if (bad) return;

    // column m of T = (I + A)^{-1} (forward substitution) and of PT = P T
    if (tid < kC) {
        const int m = tid;
        float xc[kC];
#pragma unroll
        for (int i = 0; i < kC; ++i) {
            const float *Ar = ps.A[i];
            float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
            for (int n = 0; n + 4 <= i; n += 4) {
                const float4 a4 = *reinterpret_cast<const float4 *>(Ar + n);
                s0 = fmaf(a4.x, xc[n], s0);
                s1 = fmaf(a4.y, xc[n + 1], s1);
                s2 = fmaf(a4.z, xc[n + 2], s2);
                s3 = fmaf(a4.w, xc[n + 3], s3);
            }
#pragma unroll
            for (int n = i & ~3; n < i; ++n) s0 = fmaf(Ar[n], xc[n], s0);
            xc[i] = (i == m ? 1.0f : 0.0f) - ((s0 + s1) + (s2 + s3));
        }
        float *wsb = a.ws + ((size_t)c * a.B * a.H + bh) * kWsChunkFloats;
#pragma unroll
        for (int i = 0; i < kC; ++i) {
            const float *Pr = ps.P[i];
            float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
            for (int n = 0; n + 4 <= i + 1; n += 4) {
                const float4 p4 = *reinterpret_cast<const float4 *>(Pr + n);
                s0 = fmaf(p4.x, xc[n], s0);
                s1 = fmaf(p4.y, xc[n + 1], s1);
                s2 = fmaf(p4.z, xc[n + 2], s2);
                s3 = fmaf(p4.w, xc[n + 3], s3);
            }
#pragma unroll
            for (int n = (i + 1) & ~3; n <= i; ++n) s0 = fmaf(Pr[n], xc[n], s0);
            wsb[(size_t)i * kC + m] = (s0 + s1) + (s2 + s3);   // PT row i
            wsb[(size_t)(kC + i) * kC + m] = xc[i];             // T row i
        }
    }
}

// ---------------------------------------------------------------------------
// Phase 2: the chunks of the pass in order, the state carried on the tensor core
// ---------------------------------------------------------------------------

constexpr int kEpiWarps = 4, kMmaWarp = 4, kLoadWarp = 5, kTWarp0 = 6, kTWarps = 4;
constexpr int kScanThreads = (kEpiWarps + 2 + kTWarps) * 32;

// TMEM columns (256 allocated): the three accumulators
constexpr uint32_t kColX = 0, kColOU = 64, kColS = 128;

struct ScanBars {
    uint64_t full[2], empty[2];      // input stages (TMA + cp.async)
    uint64_t t_full, t_empty;        // [PT; T] operand in shared memory
    uint64_t x_done, ou_done, s_done;  // MMA completions
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
    L.v = L.qk + 2 * kQKBytes;            // [2][8 KB] V slice, row-major [64 t][64 i]
    L.ab = L.v + 2 * kVBytes;             // [2][alpha 64, beta 64]
    L.s3 = L.ab + 2 * 512;                // [3][16 KB] S^T split (MN-major B of the X product)
    L.ru = L.s3 + 3 * 16384;              // [3][8 KB] R, then U^ (MN-major B, BF16 parts)
    L.tt = L.ru + 3 * 8192;               // [3][16 KB] [PT; T] (K-major A, BF16 parts)
    L.bytes = L.tt + 3 * 16384;
    return L;
}

__global__ void __launch_bounds__(kScanThreads, 1) chunk_scan_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, const ChunkArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
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
            mbar_init(&sb.full[s], 1);
            mbar_init(&sb.empty[s], kEpiWarps);
        }
        mbar_init(&sb.t_full, kTWarps);
        mbar_init(&sb.t_empty, 1);
        mbar_init(&sb.x_done, 1);
        mbar_init(&sb.ou_done, 1);
        mbar_init(&sb.s_done, 1);
        mbar_init(&sb.r_ready, 2);
        mbar_init(&sb.u_ready, 2);
        mbar_init(&sb.s_ready, kEpiWarps);
    }
    if (warp == kMmaWarp) tmem_alloc(&sb.tmem, 256);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = sb.tmem;

    if (warp == kLoadWarp) {
        // ---------------------------------------------------------- loader
        if (lane == 0) {
            int c = 0;
            for (; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 && !mbar_wait_bounded(&sb.empty[s], ((c >> 1) - 1) & 1)) break;
                const int tok0 = b * a.T_total + a.t0 + c * kC;
                float *ab = abbuf + s * 128;
                for (int t = 0; t < kC; ++t) {
                    cp_async4(ab + t, a.alpha + ((size_t)tok0 + t) * a.H + h);
                    cp_async4(ab + kC + t, a.beta + ((size_t)tok0 + t) * a.H + h);
                }
                cp_async_mbar_arrive(&sb.full[s]);
                mbar_arrive_expect_tx(&sb.full[s], kQKBytes + kVBytes);
                load_qk(qkbuf + s * kQKBytes, &qmap, &kmap, h, tok0, &sb.full[s]);
                tma_load_3d(vbuf + s * kVBytes, &vmap, i0, h, tok0, &sb.full[s]);
            }
            // drain copies still in flight into this CTA (after an expired wait)
            for (int j = c - 1; j >= 0 && j >= c - 2; --j) mbar_wait_bounded(&sb.full[j & 1], (j >> 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idx = idesc_bf16(128, kDVS, false, true);
            constexpr uint32_t idt = idesc_bf16(128, kDVS, false, true);
            constexpr uint32_t ids = idesc_bf16(128, kDVS, true, true);
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1, ph = c & 1;
                if (!mbar_wait_bounded(&sb.full[s], (c >> 1) & 1)) break;
                if (!mbar_wait_bounded(&sb.s_ready, ph)) break;
                tc_fence_after_sync();
                const unsigned char *qk = qkbuf + s * kQKBytes;
                // X = [Q; K] S^T, S = s0 + s1 + s2 (smallest part first)
                bool acc = false;
                for (int k16 = 0; k16 < kDK / 16; ++k16)
                    for (int p = 2; p >= 0; --p) {
                        const uint64_t bd = smem_desc(smem_u32(s3 + p * 16384 + k16 * 256), 128, 2048);
                        mma_bf16(tm + kColX, desc_qk(qk, k16), bd, idx, acc);
                        acc = true;
                    }
                mma_commit(&sb.x_done);
                if (!mbar_wait_bounded(&sb.r_ready, ph)) break;
                if (!mbar_wait_bounded(&sb.t_full, ph)) break;
                tc_fence_after_sync();
                // [O_intra; U] = [PT; T] R: parts (p, q) with p + q <= 2, smallest first
                acc = false;
                for (int k16 = 0; k16 < kC / 16; ++k16)
                    for (int n = 0; n < 6; ++n) {
                        constexpr int kP[6] = {2, 1, 0, 1, 0, 0}, kQ[6] = {0, 1, 2, 0, 1, 0};
                        const uint64_t ad = smem_desc(smem_u32(tt + kP[n] * 16384 + k16 * 4096), 2048, 128);
                        const uint64_t bd = smem_desc(smem_u32(ru + kQ[n] * 8192 + k16 * 256), 128, 1024);
                        mma_bf16(tm + kColOU, ad, bd, idt, acc);
                        acc = true;
                    }
                mma_commit(&sb.ou_done);
                mma_commit(&sb.t_empty);
                if (!mbar_wait_bounded(&sb.u_ready, ph)) break;
                tc_fence_after_sync();
                // D_S = K^T U^, U^ = u0 + u1 + u2
                acc = false;
                for (int k16 = 0; k16 < kC / 16; ++k16)
                    for (int p = 2; p >= 0; --p) {
                        const uint64_t bd = smem_desc(smem_u32(ru + p * 8192 + k16 * 256), 128, 1024);
                        mma_bf16(tm + kColS, desc_kt_mn(qk, k16), bd, ids, acc);
                        acc = true;
                    }
                mma_commit(&sb.s_done);
            }
        }
    } else if (warp >= kTWarp0) {
        // ---------------------------------------------------------- [PT; T] operand
        // row r of [PT; T] as three BF16 parts, K-major (element (r, m) of a
        // part at byte (m / 8) * 2048 + 16 r + 2 (m % 8))
        const int r = tid - kTWarp0 * 32;
        for (int c = 0; c < nc; ++c) {
            const float *src = a.ws + ((size_t)c * a.B * a.H + bh) * kWsChunkFloats + (size_t)r * kC;
            float x[kC];
#pragma unroll
            for (int q = 0; q < kC / 4; ++q) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(src) + q);
                x[4 * q] = v.x, x[4 * q + 1] = v.y, x[4 * q + 2] = v.z, x[4 * q + 3] = v.w;
            }
            if (c >= 1 && !mbar_wait_bounded(&sb.t_empty, (c - 1) & 1)) break;
#pragma unroll
            for (int g = 0; g < kC / 8; ++g) {
                __align__(16) __nv_bfloat16 p0[8], p1[8], p2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) split_bf16x3(x[8 * g + e], p0[e], p1[e], p2[e]);
                const int off = g * 2048 + 16 * r;
                *reinterpret_cast<uint4 *>(tt + off) = *reinterpret_cast<const uint4 *>(p0);
                *reinterpret_cast<uint4 *>(tt + 16384 + off) = *reinterpret_cast<const uint4 *>(p1);
                *reinterpret_cast<uint4 *>(tt + 32768 + off) = *reinterpret_cast<const uint4 *>(p2);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.t_full);
        }
    } else {
        // ---------------------------------------------------------- epilogue (warps 0..3)
        const int r = tid;                 // TMEM lane
        const int t = r & (kC - 1);        // token of this row (rows 0..63 Q / O, 64..127 K / U)
        const uint32_t ta = tm + ((uint32_t)(32 * warp) << 16);
        float S[kDVS];                     // S[i0 + i][j = r], the state slice's column r
        {
            const float *Sg = a.S + ((size_t)bh * a.DV + i0) * kDK + r;
#pragma unroll
            for (int i = 0; i < kDVS; ++i) S[i] = Sg[(size_t)i * kDK];
        }
        // write S^T (MN-major, N = value row i, K = key channel j = r) in three BF16 parts
        auto write_s3 = [&]() {
#pragma unroll
            for (int g = 0; g < kDVS / 8; ++g) {
                __align__(16) __nv_bfloat16 p0[8], p1[8], p2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) split_bf16x3(S[8 * g + e], p0[e], p1[e], p2[e]);
                const int off = g * 2048 + 16 * r;
                *reinterpret_cast<uint4 *>(s3 + off) = *reinterpret_cast<const uint4 *>(p0);
                *reinterpret_cast<uint4 *>(s3 + 16384 + off) = *reinterpret_cast<const uint4 *>(p1);
                *reinterpret_cast<uint4 *>(s3 + 32768 + off) = *reinterpret_cast<const uint4 *>(p2);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
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
                float xk[kDVS];
                tmem_load<64>(ta + kColX, xk);
                const __nv_bfloat16 *vr = reinterpret_cast<const __nv_bfloat16 *>(vbuf + s * kVBytes) + t * kDVS;
#pragma unroll
                for (int q = 0; q < kDVS / 8; ++q) {
                    // rotate the 16-byte reads so that a quarter-warp hits distinct banks
                    const int qq = (q + t) & (kDVS / 8 - 1);
                    const uint4 w = *reinterpret_cast<const uint4 *>(vr + 8 * qq);
                    const __nv_bfloat16 *vv = reinterpret_cast<const __nv_bfloat16 *>(&w);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float v = __bfloat162float(vv[e]);
                        xk[8 * qq + e] = a.delta ? v - eLt * xk[8 * qq + e] : v;
                    }
                }
#pragma unroll
                for (int g = 0; g < kDVS / 8; ++g) {
                    __align__(16) __nv_bfloat16 p0[8], p1[8], p2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) split_bf16x3(xk[8 * g + e], p0[e], p1[e], p2[e]);
                    const int off = g * 1024 + 16 * t;
                    *reinterpret_cast<uint4 *>(ru + off) = *reinterpret_cast<const uint4 *>(p0);
                    *reinterpret_cast<uint4 *>(ru + 8192 + off) = *reinterpret_cast<const uint4 *>(p1);
                    *reinterpret_cast<uint4 *>(ru + 16384 + off) = *reinterpret_cast<const uint4 *>(p2);
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.r_ready);
            }
            if (!mbar_wait_bounded(&sb.ou_done, ph)) { ok = false; break; }
            tc_fence_after_sync();
            if (r < kC) {
                // o_t = e^{L_t} (S_0 q_t) + O_intra_t, 32 value rows at a time
                __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o) +
                                    (((size_t)b * a.T_total + a.t0 + c * kC + t) * a.H + h) * a.DV + i0;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float xq[32], oi[32];
                    tmem_load<32>(ta + kColX + 32 * hf, xq);
                    tmem_load<32>(ta + kColOU + 32 * hf, oi);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        __align__(16) __nv_bfloat16 ob[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) ob[e] = __float2bfloat16_rn(fmaf(eLt, xq[8 * q + e], oi[8 * q + e]));
                        *reinterpret_cast<uint4 *>(og + 32 * hf + 8 * q) = *reinterpret_cast<const uint4 *>(ob);
                    }
                }
            } else {
                // U^_t = beta_t e^{L_C - L_t} u_t in three BF16 parts (MN-major B of K^T U^)
                float u[kDVS];
                tmem_load<64>(ta + kColOU, u);
                const float gam = be[t] * expf(LC - Lt);
#pragma unroll
                for (int g = 0; g < kDVS / 8; ++g) {
                    __align__(16) __nv_bfloat16 p0[8], p1[8], p2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) split_bf16x3(gam * u[8 * g + e], p0[e], p1[e], p2[e]);
                    const int off = g * 1024 + 16 * t;
                    *reinterpret_cast<uint4 *>(ru + off) = *reinterpret_cast<const uint4 *>(p0);
                    *reinterpret_cast<uint4 *>(ru + 8192 + off) = *reinterpret_cast<const uint4 *>(p1);
                    *reinterpret_cast<uint4 *>(ru + 16384 + off) = *reinterpret_cast<const uint4 *>(p2);
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.u_ready);
            }
            if (!mbar_wait_bounded(&sb.s_done, ph)) { ok = false; break; }
            tc_fence_after_sync();
            {
                // S_C = e^{L_C} S_0 + (U^ ^T K)^T, column r of the slice
                float ds[kDVS];
                tmem_load<64>(ta + kColS, ds);
                const float eLC = expf(LC);
#pragma unroll
                for (int i = 0; i < kDVS; ++i) S[i] = fmaf(eLC, S[i], ds[i]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.empty[s]);
            if (c + 1 < nc) write_s3();
        }
        if (ok) {
            float *Sg = a.S + ((size_t)bh * a.DV + i0) * kDK + r;
#pragma unroll
            for (int i = 0; i < kDVS; ++i) Sg[(size_t)i * kDK] = S[i];
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

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::atomic<void *> fn{nullptr};
    void *f = fn.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn.store(f, std::memory_order_release);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// A 3-D map of a BF16 activation [B*T, H, D] (innermost D): box {box_d, 1, 64}.
bool activation_map(CUtensorMap *m, const void *base, int D, int H, long long BT, int box_d) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)BT};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)box_d, 1, (cuuint32_t)kC};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t chunk_workspace_bytes(int BH, int chunks) {
    return (size_t)chunks * BH * kWsChunkFloats * sizeof(float);
}

bool chunk_path_supported(int d_k, int d_v, int gate, bool bf16) {
    return bf16 && gate == 0 && d_k == kDK && (d_v == 64 || d_v == 128);
}

cudaError_t launch_prefill_chunks(const ChunkArgs &a, const void *q, const void *k, const void *v,
                                  cudaStream_t stream) {
    if (a.nc < 1 || a.DV % kDVS != 0) return cudaErrorInvalidValue;
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
                                     scan_layout().bytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long BT = (long long)a.B * a.T_total;
    CUtensorMap qm, km, vm;
    if (!activation_map(&qm, q, kDK, a.H, BT, 8) || !activation_map(&km, k, kDK, a.H, BT, 8) ||
        !activation_map(&vm, v, a.DV, a.H, BT, kDVS))
        return cudaErrorInvalidValue;
    const int BH = a.B * a.H;
    chunk_prep_kernel<<<a.nc * BH, kPrepThreads, prep_smem_bytes(), stream>>>(qm, km, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    chunk_scan_kernel<<<BH * (a.DV / kDVS), kScanThreads, scan_layout().bytes, stream>>>(qm, km, vm, a);
    return cudaGetLastError();
}

}  // namespace lq
