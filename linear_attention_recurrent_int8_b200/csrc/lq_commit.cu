// lq_commit.cu -- the window commit on sm_100a: rebuild of the FP32 state at
// the window end, Compensator Tokens, residual smoothing and per-row
// re-quantization to 8-bit (or 6- or 4-bit) codes, or BF16 ("LeapQuant: Efficient Linear Attention with Accurate
// Recurrent State Quantization", Figure 2: the state is quantized once per
// window; Figure 4 and the Abstract: the largest outliers are kept as
// high-precision Compensator Tokens and the residual is smoothed across
// channels before the 8-bit quantization).
//
// With the running log gate L_m of each buffered record and the compensators
// taken as pseudo-records at window position 0 (they decay like S^_0):
//
//   S_n = S^_0 Diag(e^{L_n}) + [U | E_comp] [K^ | comp Diag(e^{L_n})]^T,
//   K^_m = k~_m * e^{L_n - L_m},
//
// where S^_0 = Diag(sigma) Q Diag(c) is the quantized residual of the snapshot,
// U = [u_1 .. u_n] the buffered updates and E_comp the one-hot columns of the
// compensator rows.  The rank-(n + r) term is a dense contraction and runs on
// the 5th-generation tensor core: kind::tf32 with both operands split into a
// TF32 high and low part and three products (hi*hi + hi*lo + lo*hi), which
// keeps it FP32-faithful; the accumulator lives in tensor memory (TMEM).
// Then C2-C4 (the rule stated in lq_quant.cuh) run with one value row per
// thread.  Where the rule divides (R / c_j, R' / sigma_i) this kernel
// multiplies by the FP32 inverse (1 / c_j, q / max_j |R'_ij|): one rounding
// more per element, so a code can differ by one step from the rule's where
// the quotient lies within an FP32 step of a half-integer, and sigma and c
// agree to about 1e-7 relative; the window's code tolerance (one step)
// admits it, and every element costs one product instead of a division. TMEM lane i holds row i, so row norms and row maxima are
// reductions inside a thread, and column maxima are warp reductions
// (redux.sync) plus one shared-memory pass over the four lane quarters.
//
// Structure: one persistent, warp-specialised CTA per SM walking the heads
// with a grid stride, so that loading, operand building, tensor-core work and
// quantization of consecutive heads overlap:
//  * producer (one lane): the head's records, compensators and scales into a
//    ring of shared-memory stages by 1-D bulk copies (no multicast), and an L2
//    prefetch of its codes;
//  * 4 builder warps: the TF32 hi/lo operands of the rank term into one of
//    two operand buffers;
//  * MMA warp (one lane): the MMAs of a head into one of two TMEM
//    accumulators once its operands are built and the accumulator is free;
//  * 8 epilogue warps: C1-C4 from TMEM (lane quarter q = warp % 4 holds value
//    rows 32q..32q+31, the two warps of a quarter split the key channels),
//    while the builders already work on the next head.
// Every mbarrier wait is bounded (lq_common.cuh).
#include <atomic>
#include <cstddef>

#include "lq_kernels.h"
#include "lq_quant.cuh"
#include "lq_tc.cuh"

namespace lq {
namespace {

constexpr int kEpiWarps = 8, kBldWarps = 4;
constexpr int kEpi = kEpiWarps * 32, kBld = kBldWarps * 32;
constexpr int kProducerWarp = kEpiWarps + kBldWarps, kMmaWarp = kProducerWarp + 1;
constexpr int kThreads = kEpi + kBld + 64;
constexpr int kMaxStages = 4;
constexpr int kEpiBar = 1, kBldBar = 2;  // named barriers

template <int DK, int DV>
struct alignas(16) CommitSmem {
    uint64_t full[kMaxStages], empty[kMaxStages];  // stage ring
    uint64_t ops_ready[2];                         // operand buffers filled
    uint64_t mma_done[2], tmem_free[2];            // TMEM accumulators
    uint32_t tmem;                                 // TMEM base address
    // builders
    alignas(16) float gW[DK];          // e^{L_n}, per key channel
    float dec[32];                     // scalar gate: e^{L_n - L_m}
    // epilogue
    alignas(16) float cg[DK];          // c_j e^{L_n,j}
    alignas(16) float icol[DK];        // 1 / c_j of the new snapshot
    alignas(16) float colpart[4][DK];  // column maxima per lane quarter
    float rowpart[2][128];             // row partials of the two column halves
    int comp_idx[128];                 // compensator slot of each row, -1 if none
    int sel[kMaxComp];                 // new compensator rows
};

// One stage: a head's buffered records (n of them), compensators and scales.
struct StageLayout {
    int K, U, L, comp, cs, rs, compr, bytes;
};

__host__ __device__ inline int a16(int x) { return (x + 15) & ~15; }

__host__ __device__ inline StageLayout stage_layout(int DK, int DV, int gate, int n, int R) {
    StageLayout L{};
    int o = 0;
    L.K = o;     o += a16(4 * n * DK);
    L.U = o;     o += a16(4 * n * DV);
    L.L = o;     o += a16(4 * n * (gate == 1 ? DK : 1));
    L.comp = o;  o += a16(4 * R * DK);
    L.cs = o;    o += a16(4 * DK);
    L.rs = o;    o += a16(4 * DV);
    L.compr = o; o += a16(4 * kMaxComp);
    L.bytes = (o + 127) & ~127;
    return L;
}

// Tensor-core operands (lq_tc.cuh layout): A = [U | E_comp] with 128 rows
// (value channels; zero beyond d_v) and B = [K^ | comp e^{L_n}] with d_k
// rows, K = records + compensators rounded up to 8, each as a TF32 high and
// low part.
struct OperandLayout {
    int ahi, alo, bhi, blo, kp, bytes;
};

__host__ __device__ inline OperandLayout operand_layout(int DK, int items) {
    OperandLayout L{};
    L.kp = (items + 7) & ~7;
    int o = 0;
    L.ahi = o; o += 4 * L.kp * 128;
    L.alo = o; o += 4 * L.kp * 128;
    L.bhi = o; o += 4 * L.kp * DK;
    L.blo = o; o += 4 * L.kp * DK;
    L.bytes = o;
    return L;
}

__host__ __device__ constexpr int align128(int x) { return (x + 127) & ~127; }

template <int DK, int DV>
__host__ __device__ constexpr int scratch_bytes() {
    return align128((int)sizeof(CommitSmem<DK, DV>));
}

// x rounded to TF32 (10 explicit mantissa bits), to nearest with ties away
// from zero, as a 32-bit pattern: add half a TF32 unit to the magnitude and
// truncate (a carry into the exponent is the correct rounding; the values
// here are finite).
__device__ __forceinline__ uint32_t to_tf32(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
}

// The TF32 pair (hi, lo) with x = hi + lo + O(2^-22 |x|): lo = x - hi is exact.
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

__device__ __forceinline__ uint32_t word_of(const uint4 &w, int k) {
    return k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}


// The next head of this CTA's grid-stride walk at or after `bh` that commits
// in this launch: every head with batch-synchronous positions; with
// per-sequence positions the heads of sequences whose seq_pos equals
// a.commit_match (W - 1: the window has just filled; p: a flush of the
// windows holding p records).  Every role walks the same sequence.
__device__ __forceinline__ int next_commit_head(const DecodeArgs &a, int bh) {
    const int BH = a.B * a.H;
    if (!a.seq_pos) return bh;
    for (; bh < BH; bh += gridDim.x)
        if (a.seq_pos[bh / a.H] == a.commit_match) return bh;
    return BH;
}

// FMT: the residual's storage (lq_kernels.h): codes one per byte, 4-bit codes
// two per byte (layout in lq_quant.cuh), or BF16 values.
template <int DK, int DV, int GATE, int FMT>
__global__ void __launch_bounds__(kThreads, 1) commit_kernel(const DecodeArgs a, const int NS,
                                                             const int NOPS) {
    static_assert(DV == 64 || DV == 128, "d_v must be 64 or 128");
    constexpr int NQ = DV / 32;        // lane quarters that hold rows
    constexpr int CPT = DK / 2;        // key channels per epilogue thread
    constexpr int NCH = CPT / 32;      // 32-column TMEM chunks per thread
    constexpr bool PACK4 = FMT == kCodesI4, BF16S = FMT == kCodesBF16;
    constexpr int CRB = code_row_bytes(FMT, DK);  // residual bytes per value row
    // 16-byte code words per thread, loaded one head ahead (a BF16 row half
    // is loaded chunk by chunk where it is used instead)
    constexpr int NCW = PACK4 ? CPT / 32 : BF16S ? 1 : CPT / 16;
    constexpr int JB = CRB / (DK / 2);  // residual bytes per 2 key channels
    constexpr int G = GATE == 1 ? DK : 1;
    extern __shared__ __align__(128) unsigned char smem[];
    auto &cs = *reinterpret_cast<CommitSmem<DK, DV> *>(smem);
    const int nrec = a.pos, R = a.R, W = a.W, BH = a.B * a.H;
    const StageLayout SL = stage_layout(DK, DV, GATE, nrec, R);
    const OperandLayout OL = operand_layout(DK, nrec + R);
    unsigned char *stages = smem + scratch_bytes<DK, DV>();
    unsigned char *opsbase = stages + (size_t)NS * SL.bytes;
    const int Kp = OL.kp;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0) tmem_alloc(&cs.tmem, 2 * DK);  // two FP32 accumulators of d_k columns
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&cs.full[s], 1);
            mbar_init(&cs.empty[s], kEpiWarps + kBldWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&cs.ops_ready[b], kBldWarps);
            mbar_init(&cs.mma_done[b], 1);
            mbar_init(&cs.tmem_free[b], kEpiWarps);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    // ------------------------------------------------------------ producer
    if (warp == kProducerWarp) {
        if (lane == 0) {
            int it = 0;
            for (int bh = next_commit_head(a, blockIdx.x); bh < BH; bh = next_commit_head(a, bh + gridDim.x), ++it) {
                const int s = it % NS;
                if (it >= NS && !mbar_wait_bounded(&cs.empty[s], ((it / NS) - 1) & 1)) break;
                unsigned char *st = stages + (size_t)s * SL.bytes;
                if (GATE == 0)
                    for (int m = 0; m < nrec; ++m) cp_async4(st + SL.L + 4 * m, a.buf_gate + (size_t)bh * W + m);
                for (int c = 0; c < R; ++c) cp_async4(st + SL.compr + 4 * c, a.comp_row + (size_t)bh * R + c);
                cp_async_mbar_arrive(&cs.full[s]);
                const uint32_t bytes = 4 * nrec * (DK + DV) + (GATE == 1 ? 4 * nrec * DK : 0) + 4 * R * DK +
                                       4 * DK + 4 * DV;
                mbar_arrive_expect_tx(&cs.full[s], bytes);
                bulk_g2s(st + SL.K, a.buf_k + (size_t)bh * W * DK, 4 * nrec * DK, &cs.full[s]);
                bulk_g2s(st + SL.U, a.buf_u + (size_t)bh * W * DV, 4 * nrec * DV, &cs.full[s]);
                if (GATE == 1) bulk_g2s(st + SL.L, a.buf_gate + (size_t)bh * W * DK, 4 * nrec * DK, &cs.full[s]);
                if (R > 0) bulk_g2s(st + SL.comp, a.comp_val + (size_t)bh * R * DK, 4 * R * DK, &cs.full[s]);
                bulk_g2s(st + SL.cs, a.col_smooth + (size_t)bh * DK, 4 * DK, &cs.full[s]);
                bulk_g2s(st + SL.rs, a.row_scale + (size_t)bh * DV, 4 * DV, &cs.full[s]);
                prefetch_l2(a.codes + (size_t)bh * DV * CRB, DV * CRB);
            }
        }
        return;
    }

    // ------------------------------------------------------------ MMA issuer
    if (warp == kMmaWarp) {
        if (lane == 0) {
            int it = 0;
            for (int bh = next_commit_head(a, blockIdx.x); bh < BH; bh = next_commit_head(a, bh + gridDim.x), ++it) {
                const int b = it & 1, ob = it % NOPS;
                if (!mbar_wait_bounded(&cs.ops_ready[ob], (it / NOPS) & 1)) break;
                // the accumulator is free once the epilogue of head it - 2 is done
                if (it >= 2 && !mbar_wait_bounded(&cs.tmem_free[b], ((it - 2) >> 1) & 1)) break;
                tc_fence_after_sync();
                const unsigned char *ops = opsbase + (size_t)ob * OL.bytes;
                constexpr uint32_t idesc = idesc_tf32(128, DK);
                const uint32_t d = cs.tmem + b * DK;
                const uint32_t ah = smem_u32(ops + OL.ahi), al = smem_u32(ops + OL.alo);
                const uint32_t bhs = smem_u32(ops + OL.bhi), bls = smem_u32(ops + OL.blo);
                for (int k8 = 0; k8 < Kp / 8; ++k8) {
                    const uint32_t ao = k8 * 2 * 128 * 16, bo = k8 * 2 * DK * 16;
                    const uint64_t dah = smem_desc(ah + ao, 128 * 16, 128);
                    const uint64_t dal = smem_desc(al + ao, 128 * 16, 128);
                    const uint64_t dbh = smem_desc(bhs + bo, DK * 16, 128);
                    const uint64_t dbl = smem_desc(bls + bo, DK * 16, 128);
                    mma_tf32(d, dah, dbl, idesc, k8 > 0);
                    mma_tf32(d, dal, dbh, idesc, true);
                    mma_tf32(d, dah, dbh, idesc, true);
                }
                mma_commit(&cs.mma_done[b]);
            }
        }
        return;
    }

    // ------------------------------------------------------------ builders
    if (warp >= kEpiWarps) {
        const int bt = tid - kEpi;
        int it = 0;
        for (int bh = next_commit_head(a, blockIdx.x); bh < BH; bh = next_commit_head(a, bh + gridDim.x), ++it) {
            const int s = it % NS;
            bool ok = mbar_wait_bounded(&cs.full[s], (it / NS) & 1);
            // the operand buffer is free once the MMAs that read it completed
            if (ok && it >= NOPS) ok = mbar_wait_bounded(&cs.mma_done[(it - NOPS) & 1], ((it - NOPS) >> 1) & 1);
            if (named_sync_or<kBldBar, kBld>(!ok)) break;  // the group leaves together
            const unsigned char *st = stages + (size_t)s * SL.bytes;
            const float *Ks = reinterpret_cast<const float *>(st + SL.K);
            const float *Us = reinterpret_cast<const float *>(st + SL.U);
            const float *Ls = reinterpret_cast<const float *>(st + SL.L);
            const float *Cs = reinterpret_cast<const float *>(st + SL.comp);
            const int *Cr = reinterpret_cast<const int *>(st + SL.compr);
            unsigned char *ops = opsbase + (size_t)(it % NOPS) * OL.bytes;
            unsigned char *Ahi = ops + OL.ahi, *Alo = ops + OL.alo, *Bhi = ops + OL.bhi, *Blo = ops + OL.blo;
            for (int j = bt; j < DK; j += kBld) cs.gW[j] = expf(Ls[(nrec - 1) * G + (GATE == 1 ? j : 0)]);
            if (GATE == 0 && bt < nrec) cs.dec[bt] = expf(Ls[nrec - 1] - Ls[bt]);
            named_sync<kBldBar, kBld>();
            // B: row j = key channel, element m = record m or compensator m - n.
            // Every load is issued unconditionally from a clamped index (all
            // inside the stage) and the element chosen by selects, so the
            // loads of a slab are in flight together.
            {
                constexpr int SPJ = kBld / DK;        // threads per key channel
                const int j = bt % DK;
                const float Lnj = GATE == 1 ? Ls[(nrec - 1) * DK + j] : 0.0f;
                const float gj = cs.gW[j];
                for (int kc = bt / DK; kc < Kp / 4; kc += SPJ) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int m = 4 * kc + e;
                        const int mr = m < nrec ? m : nrec - 1;
                        const int mc = m - nrec < 0 ? 0 : (m - nrec < R ? m - nrec : (R > 0 ? R - 1 : 0));
                        const float dcy = GATE == 1 ? expf(Lnj - Ls[mr * DK + j]) : cs.dec[mr];
                        const float xr = Ks[mr * DK + j] * dcy;
                        const float xc = R > 0 ? Cs[mc * DK + j] * gj : 0.0f;
                        const float x = m < nrec ? xr : (m < nrec + R ? xc : 0.0f);
                        split_tf32(x, hi[e], lo[e]);
                    }
                    const int off = (kc * DK + j) * 16;
                    *reinterpret_cast<uint4 *>(Bhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(Blo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
            // A: row r = value channel (zero beyond d_v), element m = u_m,r or
            // the compensator's one-hot column (exact in TF32)
            {
                const int r = bt;
                const int rr = r < DV ? r : DV - 1;
                for (int kc = 0; kc < Kp / 4; ++kc) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int m = 4 * kc + e;
                        const int mr = m < nrec ? m : nrec - 1;
                        const int mc = m - nrec < 0 ? 0 : (m - nrec < R ? m - nrec : (R > 0 ? R - 1 : 0));
                        const float xu = Us[mr * DV + rr];
                        const float xe = (R > 0 && Cr[mc] == r) ? 1.0f : 0.0f;
                        float x = m < nrec ? xu : (m < nrec + R ? xe : 0.0f);
                        if (r >= DV) x = 0.0f;
                        split_tf32(x, hi[e], lo[e]);
                    }
                    const int off = (kc * 128 + r) * 16;
                    *reinterpret_cast<uint4 *>(Ahi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(Alo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&cs.ops_ready[it % NOPS]);
                mbar_arrive(&cs.empty[s]);
            }
        }
        return;
    }

    // ------------------------------------------------------------ epilogue
    const int qtr = warp & 3, half = warp >> 2;
    const bool has_row = qtr < NQ;  // warp-uniform
    const int row = 32 * qtr + lane, j0 = half * CPT;
    // the row half's old codes, loaded one head ahead (the producer has
    // prefetched them into L2)
    uint4 cw[NCW], cw_next[NCW];
    auto load_codes = [&](int bhx, uint4(&dst)[NCW]) {
        if (!BF16S && has_row && bhx < BH) {
            const int8_t *src = a.codes + ((size_t)bhx * DV + row) * CRB + j0 * JB / 2;
#pragma unroll
            for (int c = 0; c < NCW; ++c) dst[c] = *reinterpret_cast<const uint4 *>(src + 16 * c);
        }
    };
    load_codes(next_commit_head(a, blockIdx.x), cw_next);
    int it = 0;
    for (int bh = next_commit_head(a, blockIdx.x); bh < BH; bh = next_commit_head(a, bh + gridDim.x), ++it) {
        const int s = it % NS, b = it & 1;
        const bool okf = mbar_wait_bounded(&cs.full[s], (it / NS) & 1);
        if (named_sync_or<kEpiBar, kEpi>(!okf)) break;  // the group leaves together
        const unsigned char *st = stages + (size_t)s * SL.bytes;
        const float *Ls = reinterpret_cast<const float *>(st + SL.L);
        const float *Css = reinterpret_cast<const float *>(st + SL.cs);
        const float *Rss = reinterpret_cast<const float *>(st + SL.rs);
        int8_t *codes_row = a.codes + ((size_t)bh * DV + (has_row ? row : 0)) * CRB + j0 * JB / 2;
        const uint32_t tq = cs.tmem + ((uint32_t)(32 * qtr) << 16) + b * DK + j0;
        for (int j = tid; j < DK; j += kEpi) cs.cg[j] = Css[j] * expf(Ls[(nrec - 1) * G + (GATE == 1 ? j : 0)]);
        if (tid < DV) cs.comp_idx[tid] = -1;
#pragma unroll
        for (int c = 0; c < NCW; ++c) cw[c] = cw_next[c];
        load_codes(next_commit_head(a, bh + gridDim.x), cw_next);
        const float sig = has_row ? Rss[row] : 0.0f;
        const bool ok = mbar_wait_bounded(&cs.mma_done[b], (it >> 1) & 1);
        if (named_sync_or<kEpiBar, kEpi>(!ok)) break;  // also publishes cg and comp_idx
        tc_fence_after_sync();

        // C1: boundary term added to the rank term; squared row norm
        if (has_row) {
            float2 ss = make_float2(0.0f, 0.0f);
            const float2 sg2 = make_float2(sig, sig);
            const float2 off2 = make_float2(-8388736.0f, -8388736.0f);
            // 4-bit: each biased byte is 16 Q + 128; x / 16 - (2^23 + 128) / 16 = Q exactly
            const float2 sixteenth2 = make_float2(0.0625f, 0.0625f);
            const float2 off16_2 = make_float2(-524296.0f, -524296.0f);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float x[32];
                uint4 bw[BF16S ? 4 : 1];  // BF16: this chunk's 32 values (64 bytes)
                if constexpr (BF16S) {
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        bw[v] = *reinterpret_cast<const uint4 *>(codes_row + 64 * c + 16 * v);
                }
                tmem_load<32>(tq + 32 * c, x);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if constexpr (BF16S) {
                        // BF16 -> FP32 is a 16-bit shift; sigma = c = 1
                        const uint32_t wa = word_of(bw[q / 2], 2 * (q % 2));
                        const uint32_t wb = word_of(bw[q / 2], 2 * (q % 2) + 1);
                        const float4 g = *reinterpret_cast<const float4 *>(cs.cg + j0 + 32 * c + 4 * q);
                        const float2 f01 = make_float2(__uint_as_float(wa << 16), __uint_as_float(wa & 0xFFFF0000u));
                        const float2 f23 = make_float2(__uint_as_float(wb << 16), __uint_as_float(wb & 0xFFFF0000u));
                        const float2 y01 = __ffma2_rn(f01, make_float2(g.x, g.y), make_float2(x[4 * q], x[4 * q + 1]));
                        const float2 y23 = __ffma2_rn(f23, make_float2(g.z, g.w), make_float2(x[4 * q + 2], x[4 * q + 3]));
                        ss = __ffma2_rn(y01, y01, ss);
                        ss = __ffma2_rn(y23, y23, ss);
                        x[4 * q] = y01.x;
                        x[4 * q + 1] = y01.y;
                        x[4 * q + 2] = y23.x;
                        x[4 * q + 3] = y23.y;
                    } else {
                        uint32_t cword;
                        if constexpr (PACK4) {
                            // channels 8h..8h+3 sit in the low nibbles of word h,
                            // 8h+4..8h+7 in the high ones: move the nibble into
                            // the high half of each byte, giving 16 Q as an int8
                            const uint32_t w = word_of(cw[c], q / 2);
                            cword = (q & 1) ? (w & 0xF0F0F0F0u) : ((w << 4) & 0xF0F0F0F0u);
                        } else {
                            cword = word_of(cw[2 * c + q / 4], q % 4);
                        }
                        const uint32_t u = cword ^ 0x80808080u;
                        const float4 g = *reinterpret_cast<const float4 *>(cs.cg + j0 + 32 * c + 4 * q);
                        // code + 128 in the low mantissa bits of 2^23, minus (2^23 + 128)
                        float2 f01 = make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)),
                                                 __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)));
                        float2 f23 = make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)),
                                                 __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653)));
                        if constexpr (PACK4) {
                            f01 = __fmul2_rn(__ffma2_rn(f01, sixteenth2, off16_2), sg2);
                            f23 = __fmul2_rn(__ffma2_rn(f23, sixteenth2, off16_2), sg2);
                        } else {
                            f01 = __fmul2_rn(__fadd2_rn(f01, off2), sg2);
                            f23 = __fmul2_rn(__fadd2_rn(f23, off2), sg2);
                        }
                        const float2 y01 = __ffma2_rn(f01, make_float2(g.x, g.y), make_float2(x[4 * q], x[4 * q + 1]));
                        const float2 y23 = __ffma2_rn(f23, make_float2(g.z, g.w), make_float2(x[4 * q + 2], x[4 * q + 3]));
                        ss = __ffma2_rn(y01, y01, ss);
                        ss = __ffma2_rn(y23, y23, ss);
                        x[4 * q] = y01.x;
                        x[4 * q + 1] = y01.y;
                        x[4 * q + 2] = y23.x;
                        x[4 * q + 3] = y23.y;
                    }
                }
                tmem_store32(tq + 32 * c, x);
            }
            cs.rowpart[half][row] = ss.x + ss.y;
            tmem_wait_st();
        }
        named_sync<kEpiBar, kEpi>();

        // C2: warp 0 selects the R rows of largest squared norm, ties to the
        // smaller row.  Keys are the norm's bit pattern + 1 (non-negative
        // floats order like their bits); a selected row's key becomes 0.
        if (warp == 0 && R > 0) {
            uint32_t key[NQ];
#pragma unroll
            for (int p = 0; p < NQ; ++p)
                key[p] = __float_as_uint(cs.rowpart[0][lane + 32 * p] + cs.rowpart[1][lane + 32 * p]) + 1u;
            for (int c = 0; c < R; ++c) {
                uint32_t km = key[0];
#pragma unroll
                for (int p = 1; p < NQ; ++p) km = km > key[p] ? km : key[p];
                km = __reduce_max_sync(0xffffffffu, km);
                uint32_t mine = DV;
#pragma unroll
                for (int p = NQ - 1; p >= 0; --p)
                    if (key[p] == km) mine = lane + 32 * p;
                const uint32_t bi = __reduce_min_sync(0xffffffffu, mine);
#pragma unroll
                for (int p = 0; p < NQ; ++p)
                    if (lane + 32 * p == (int)bi) key[p] = 0u;
                if (lane == 0) {
                    cs.sel[c] = bi;
                    cs.comp_idx[bi] = c;
                }
            }
        }
        named_sync<kEpiBar, kEpi>();

        // compensator rows leave the residual exactly (written out, zeroed in
        // TMEM); C3 (1/2): column maxima of |R| per lane quarter
        if (tid < R) a.comp_row[(size_t)bh * R + tid] = cs.sel[tid];
        if (has_row) {
            const int cidx = cs.comp_idx[row];
            const bool any_comp = __any_sync(0xffffffffu, cidx >= 0);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float x[32];
                tmem_load<32>(tq + 32 * c, x);
                if (any_comp) {
                    if (cidx >= 0) {
                        float *dst = a.comp_val + ((size_t)bh * R + cidx) * DK + j0 + 32 * c;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = 0.0f;
                    }
                    __syncwarp();
                    tmem_store32(tq + 32 * c, x);
                }
                if constexpr (!BF16S) {  // BF16: no smoothing, no column maxima
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 m = make_float4(warp_max_abs(x[e]), warp_max_abs(x[e + 1]),
                                                     warp_max_abs(x[e + 2]), warp_max_abs(x[e + 3]));
                        if (lane == 0) *reinterpret_cast<float4 *>(&cs.colpart[qtr][j0 + 32 * c + e]) = m;
                    }
                }
            }
            if (any_comp) tmem_wait_st();
        }
        named_sync<kEpiBar, kEpi>();
        // C3 (2/2): smoothing factor c_j and its inverse
        for (int j = tid; j < DK; j += kEpi) {
            float mj = 0.0f;
            if constexpr (!BF16S) {
                mj = cs.colpart[0][j];
#pragma unroll
                for (int q = 1; q < NQ; ++q) mj = fmaxf(mj, cs.colpart[q][j]);
            }
            const float c = (a.smoothing && mj > 0.0f) ? __fsqrt_rn(mj) : 1.0f;
            a.col_smooth[(size_t)bh * DK + j] = c;
            cs.icol[j] = __fdiv_rn(1.0f, c);
        }
        named_sync<kEpiBar, kEpi>();

        // BF16 residual: unit scale and the values rounded to BF16 (nearest even)
        if constexpr (BF16S) {
            if (has_row) {
                if (half == 0) a.row_scale[(size_t)bh * DV + row] = 1.0f;
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    float x[32];
                    tmem_load<32>(tq + 32 * c, x);
                    uint32_t hv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const __nv_bfloat162 p = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
                        hv[e] = *reinterpret_cast<const uint32_t *>(&p);
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        *reinterpret_cast<uint4 *>(codes_row + 64 * c + 16 * v) =
                            make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2], hv[4 * v + 3]);
                }
            }
        }
        // C4: R' = R (1/c) (kept in TMEM) and its row maximum
        if (!BF16S && has_row) {
            float mx = 0.0f;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float x[32];
                tmem_load<32>(tq + 32 * c, x);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 ic = *reinterpret_cast<const float4 *>(cs.icol + j0 + 32 * c + e);
                    const float2 y01 = __fmul2_rn(make_float2(x[e], x[e + 1]), make_float2(ic.x, ic.y));
                    const float2 y23 = __fmul2_rn(make_float2(x[e + 2], x[e + 3]), make_float2(ic.z, ic.w));
                    x[e] = y01.x;
                    x[e + 1] = y01.y;
                    x[e + 2] = y23.x;
                    x[e + 3] = y23.y;
                    mx = max3(mx, fabsf(y01.x), fabsf(y01.y));
                    mx = max3(mx, fabsf(y23.x), fabsf(y23.y));
                }
                tmem_store32(tq + 32 * c, x);
            }
            cs.rowpart[half][row] = mx;
            tmem_wait_st();
        }
        named_sync<kEpiBar, kEpi>();
        // C4: sigma = max / q and the codes (q = 127, 31 or 7).  |R'_ij| <=
        // max_j |R'_ij| makes |R'_ij * (q / max)| <= q (1 + 2^-23), which
        // rounds to at most q: no clamp.  The magic-number addition rounds
        // half to even; the low byte of its bits is the two's-complement code
        // (its low nibble the 4-bit code).
        if (!BF16S && has_row) {
            const float qmax = (float)((1 << (a.bits - 1)) - 1);  // 127, 31 or 7
            const float mxr = fmaxf(cs.rowpart[0][row], cs.rowpart[1][row]);
            if (half == 0) a.row_scale[(size_t)bh * DV + row] = __fdiv_rn(mxr, qmax);
            const float inv = mxr > 0.0f ? __fdiv_rn(qmax, mxr) : 0.0f;
            const float2 inv2 = make_float2(inv, inv), mg2 = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float x[32];
                tmem_load<32>(tq + 32 * c, x);
                uint32_t wv[8];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float2 y01 = __fadd2_rn(__fmul2_rn(make_float2(x[4 * g], x[4 * g + 1]), inv2), mg2);
                    const float2 y23 = __fadd2_rn(__fmul2_rn(make_float2(x[4 * g + 2], x[4 * g + 3]), inv2), mg2);
                    wv[g] = __byte_perm(__byte_perm(__float_as_uint(y01.x), __float_as_uint(y01.y), 0x0040),
                                        __byte_perm(__float_as_uint(y23.x), __float_as_uint(y23.y), 0x0040),
                                        0x5410);
                }
                if constexpr (PACK4) {
                    // word h: channels 8h..8h+3 low nibbles, 8h+4..8h+7 high
                    uint32_t pw[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        pw[h] = (wv[2 * h] & 0x0F0F0F0Fu) | ((wv[2 * h + 1] & 0x0F0F0F0Fu) << 4);
                    *reinterpret_cast<uint4 *>(codes_row + 16 * c) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
                } else {
                    *reinterpret_cast<uint4 *>(codes_row + 32 * c) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    *reinterpret_cast<uint4 *>(codes_row + 32 * c + 16) = make_uint4(wv[4], wv[5], wv[6], wv[7]);
                }
            }
        }
        // this head's TMEM reads are complete: release the accumulator and the stage
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&cs.tmem_free[b]);
            mbar_arrive(&cs.empty[s]);
        }
    }
    tc_fence_before_sync();
    named_sync<kEpiBar, kEpi>();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(cs.tmem, 2 * DK);
    }
}

// Per-device launch constants.
struct DeviceInfo {
    int sms, smem_optin;
};

template <int DK, int DV, int GATE, int FMT>
cudaError_t launch_c(const DecodeArgs &a, cudaStream_t stream) {
    static std::atomic<uint64_t> configured{0};  // devices already set up
    static DeviceInfo info[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = commit_kernel<DK, DV, GATE, FMT>;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        DeviceInfo I{};
        e = cudaDeviceGetAttribute(&I.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, I.smem_optin);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&I.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        info[dev & 63] = I;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const DeviceInfo &I = info[dev & 63];
    const StageLayout SL = stage_layout(DK, DV, GATE, a.pos, a.R);
    const OperandLayout OL = operand_layout(DK, a.pos + a.R);
    const int fixed = scratch_bytes<DK, DV>();
    // two operand buffers when they fit next to two stages, then as many
    // stages as fit (up to four)
    int nops = 2;
    if (fixed + 2 * OL.bytes + 2 * SL.bytes > I.smem_optin) nops = 1;
    int ns = (I.smem_optin - fixed - nops * OL.bytes) / SL.bytes;
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 1) return cudaErrorInvalidConfiguration;
    const int smem = fixed + ns * SL.bytes + nops * OL.bytes;
    const int BH = a.B * a.H;
    const int grid = BH < I.sms ? BH : I.sms;
    kern<<<grid, kThreads, smem, stream>>>(a, ns, nops);
    return cudaGetLastError();
}
template <int DK, int DV>
cudaError_t launch_c_d(const DecodeArgs &a, int gate, cudaStream_t stream) {
    const int fmt = code_format(a.bits);
    if (fmt == kCodesI4)
        return gate == 1 ? launch_c<DK, DV, 1, kCodesI4>(a, stream) : launch_c<DK, DV, 0, kCodesI4>(a, stream);
    if (fmt == kCodesBF16)
        return gate == 1 ? launch_c<DK, DV, 1, kCodesBF16>(a, stream)
                         : launch_c<DK, DV, 0, kCodesBF16>(a, stream);
    return gate == 1 ? launch_c<DK, DV, 1, kCodesI8>(a, stream) : launch_c<DK, DV, 0, kCodesI8>(a, stream);
}

}  // namespace

namespace {
__global__ void advance_positions_kernel(int32_t *seq_pos, int B, int W) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) {
        const int p = seq_pos[b];
        if (p >= 0 && p < W) seq_pos[b] = p + 1 == W ? 0 : p + 1;
    }
}
}  // namespace

namespace {
__global__ void reset_positions_kernel(int32_t *seq_pos, int B, int W) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) {
        const int p = seq_pos[b];
        if (p > 0 && p < W) seq_pos[b] = 0;
        if (p >= W) atomicOr(&g_dev_error, kErrBadPosition);
    }
}
}  // namespace

cudaError_t launch_advance_positions(int32_t *seq_pos, int B, int W, cudaStream_t stream) {
    advance_positions_kernel<<<(B + 255) / 256, 256, 0, stream>>>(seq_pos, B, W);
    return cudaGetLastError();
}

cudaError_t launch_reset_positions(int32_t *seq_pos, int B, int W, cudaStream_t stream) {
    reset_positions_kernel<<<(B + 255) / 256, 256, 0, stream>>>(seq_pos, B, W);
    return cudaGetLastError();
}

cudaError_t launch_commit(const DecodeArgs &a, int d_k, int d_v, int gate, cudaStream_t stream) {
    if (a.pos < 1 || a.pos > 32 || a.R < 0 || a.R > kMaxComp) return cudaErrorInvalidValue;
    if (a.bits != 8 && a.bits != 6 && a.bits != 4 && a.bits != 16) return cudaErrorInvalidValue;
    if (a.comp_u && a.R > 0) return launch_svd_commit(a, d_k, d_v, gate, stream);
    if (d_k == 128 && d_v == 128) return launch_c_d<128, 128>(a, gate, stream);
    if (d_k == 128 && d_v == 64) return launch_c_d<128, 64>(a, gate, stream);
    if (d_k == 64 && d_v == 128) return launch_c_d<64, 128>(a, gate, stream);
    if (d_k == 64 && d_v == 64) return launch_c_d<64, 64>(a, gate, stream);
    return cudaErrorInvalidValue;
}

}  // namespace lq
