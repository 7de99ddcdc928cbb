// lq_decode.cu -- per-window decode from a quantized state on sm_100a.
//
// "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
// Quantization", Figure 2: within a window the int8 boundary state S^_0 stays
// fixed and each token's update is buffered in FP32; the output of token t is
// computed from S^_0 together with the buffered updates.  With
// u_t = v_t - S_{t-1} b_t (equation 1, Appendix Table 4) and the gate kept as
// a running log L_t:
//
//   S_{t-1} b_t = S^_0 (e^{L_t} * k_t) + sum_{m<t} u_m (k~_m * e^{L_t - L_m}) . k_t
//   o_t         = S^_0 (e^{L_t} * q_t) + sum_{m<t} u_m (k~_m * e^{L_t - L_m}) . q_t
//                 + u_t (k~_t . q_t)
//
// (D_{1..t-1} b_t = e^{L_{t-1}} alpha_t k_t = e^{L_t} k_t for both gate kinds;
// e^{x} is per key channel for the diagonal gate.)  Compensator Tokens are
// pseudo-records at window position 0 (Figure 4; they share the update path
// of real tokens), so they enter with decay e^{L_t}: record (e_row, comp_val)
// under the row rule, (u_c, k~_c) under the SVD rule (lq_svd.cu).
//
// The boundary state's residual is stored as 8-bit (or 6-bit) codes one per
// byte, 4-bit codes two per byte (layout in lq_quant.cuh), or BF16 values
// (the format FMT of lq_kernels.h).
//
// Kernel structure (persistent, warp-specialised, 12 warps per CTA):
//  * the grid walks the (sequence, head) pairs with a grid stride; each head
//    goes through a ring of shared-memory stages;
//  * producer (warp 8, one lane): streams the head's codes, scales,
//    smoothing factors, compensators, buffered records and the first token's
//    q/k/v into a stage with 1-D bulk copies (no multicast) -> "full";
//  * prep A (warp 9): for every token of the call, the vectors
//    x_k = c e^L k and x_q = c e^L q split into three int8 limbs per
//    16-channel chunk (kept in FP32 for a BF16 residual), and k~_t . q_t
//    -> "prepared";
//  * prep B (warps 10, 11): the records (L_t, k~_t) of the new tokens and
//    every coefficient (k~_m e^{L_t-L_m}) . k_t, . q_t of the buffered records
//    and compensators -> "prepared";
//  * consumers (warps 0-7): warp w owns value rows [w*d_v/8, (w+1)*d_v/8).  It
//    forms S^_0 x for its rows (dp4a of the codes with the limbs, FP32
//    combine, transposing warp reduction), then u_t and o_t for the same rows
//    from the coefficients and its own buffered u.  No CTA barrier is needed
//    per head; the consumers release the stage through "empty".  With b = 0
//    (delta = 0) the x_k side is neither split nor multiplied.
// The window commit is a separate kernel (lq_commit.cu).
// Every wait is bounded (lq_common.cuh); a wait that expires sets the device
// error word and the waiting warp stops.
#include <atomic>
#include <cstddef>
#include <type_traits>

#include "lq_kernels.h"
#include "lq_quant.cuh"
#include "lq_tc.cuh"

namespace lq {

__device__ unsigned int g_dev_error = 0;

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kProducerWarp = 8, kPrepAWarp = 9, kPrepBWarp = 10, kPrepBWarps = 2;
constexpr int kPrepWarps = 1 + kPrepBWarps;
constexpr int kThreads = (kConsumerWarps + 1 + kPrepWarps) * 32;
constexpr int kMaxStages = 8;
constexpr int kCoef = 32 + kMaxComp + 1;

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }

// Per-token results of the prep warps inside a stage.
struct PrepLayout {
    int limb, lscale, coefA, coefG, bytes;
};

__host__ __device__ inline PrepLayout prep_layout(int DK, int fmt, bool tc = false) {
    PrepLayout P{};
    int o = 0;
    P.limb = o;                            // int8 [6][DK]: x_k limbs 0..2, x_q limbs 0..2,
                                           // or (BF16 residual) float [2][DK]: x_k, x_q;
                                           // none with the tensor-core matvec (the limbs
                                           // are the stage's B operand)
    o += tc ? 0 : fmt == kCodesBF16 ? 8 * DK : 6 * DK;
    P.lscale = o; o += 16;                 // float [2]: scales of x_k, x_q
    P.coefA = o;  o += align16(4 * kCoef);  // records, compensators (16-byte aligned)
    P.coefG = o;  o += align16(4 * kCoef);  // records, compensators, own token (k~.q)
    P.bytes = align16(o);
    return P;
}

// Byte offsets inside one stage (one head's operands).  `nrec` is the number
// of record slots the stage holds (records read plus records written), `n`
// the number of tokens of the call; `fmt` the residual's storage.
struct StageLayout {
    int codes, bop, sig, cs, compv, compr, compu, recK, recU, recL, q, k, v, al, scal, prep, bytes;
};

// Rows of the tensor-core matvec's B operand for n tokens: 8 per token (x_k
// limbs 0..2, x_q limbs 0..2, two unused), N = 8 for one token, else a
// multiple of 16 (the kind::i8 shapes with M = 128).
__host__ __device__ constexpr int tc_rows(int n) { return n == 1 ? 8 : 16 * ((n + 1) / 2); }

// With tc (tensor-core matvec) the codes and the B operand are not part of
// the stage (they live in a separate 1024-byte aligned array, tc_tile_bytes
// per stage) and codes = bop = -1.
// ru: rows of rank-one compensator vectors u_c (R with the SVD rule, else 0).
__host__ __device__ inline StageLayout stage_layout(int DK, int DV, int gate, int R, int nrec,
                                                   int n, int e, int fmt, bool tc = false,
                                                   int ru = 0) {
    StageLayout L{};
    int o = 0;
    L.codes = tc ? -1 : o;
    o += tc ? 0 : align16(DV * code_row_bytes(fmt, DK));
    L.bop = -1;
    L.sig = o;   o += align16(4 * DV);
    L.cs = o;    o += align16(4 * DK);
    L.compv = o; o += align16(4 * R * DK);
    L.compr = o; o += align16(4 * kMaxComp);
    L.compu = o; o += align16(4 * ru * DV);
    L.recK = o;  o += align16(4 * nrec * DK);
    L.recU = o;  o += align16(4 * nrec * DV);
    L.recL = o;  o += align16(4 * nrec * (gate == 1 ? DK : 1));
    L.q = o;     o += align16(e * DK);
    L.k = o;     o += align16(e * DK);
    L.v = o;     o += align16(e * DV);
    L.al = o;    o += gate == 1 ? align16(4 * DK) : 0;
    L.scal = o;  o += 16;                  // float: alpha (scalar gate), beta of token 0
    L.prep = o;  o += n * prep_layout(DK, fmt, tc).bytes;
    L.bytes = align16(o);
    return L;
}

// Bytes of one stage's tensor-core tile: the 128 x 128 codes (128-byte
// swizzle) and the B operand of n tokens; a multiple of 1024.
__host__ __device__ constexpr int tc_tile_bytes(int n) { return 128 * 128 + 128 * tc_rows(n); }

__host__ __device__ constexpr int header_bytes() { return 3 * kMaxStages * 8; }

// Splits the d_k-vector x (lane l holds x_j for the CPL channels
// j = j0 .. j0+CPL-1) into NL int8 limbs with one scale s = max_j |x_j| / 127:
// x ~= s (X0 + X1/2^7 [+ X2/2^14]), |error| <= s / 2^(7 NL - 6) (plus FP32
// rounding).  Writes limb l as row row0 + l of `limb` -- plain rows of DK
// bytes, or (SW128, d_k = 128) the rows of a K-major operand with the
// 128-byte swizzle -- and *lscale = s * post (post: a factor of the vector
// that was left out of x, such as a scalar gate).
template <int CPL, int NL, bool SW128 = false>
__device__ __forceinline__ void split_limbs(const float (&x)[CPL], int8_t *limb, int DK,
                                            float *lscale, int j0, int row0, float post = 1.0f) {
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) m = fmaxf(m, fabsf(x[e]));
    m = group_max<32>(m);
    const float inv = m > 0.0f ? __fdiv_rn(127.0f, m) : 0.0f;
    uint32_t w[NL];
#pragma unroll
    for (int l = 0; l < NL; ++l) w[l] = 0;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        float r = x[e] * inv;
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            const float xl = rintf(r);
            w[l] |= (static_cast<uint32_t>(static_cast<int>(xl)) & 0xFFu) << (8 * e);
            r = (r - xl) * 128.0f;
        }
    }
#pragma unroll
    for (int l = 0; l < NL; ++l) {
        const int r = row0 + l;
        if constexpr (SW128) {
            static_assert(CPL == 4, "the swizzled operand has d_k = 128");
            const int off = (r >> 3) * 1024 + (r & 7) * 128 + ((((j0 >> 4) ^ r) & 7) << 4) + (j0 & 15);
            *reinterpret_cast<uint32_t *>(limb + off) = w[l];
        } else if constexpr (CPL == 4) {
            *reinterpret_cast<uint32_t *>(limb + r * DK + j0) = w[l];
        } else {
            *reinterpret_cast<uint16_t *>(limb + r * DK + j0) = (uint16_t)w[l];
        }
    }
    if (threadIdx.x % 32 == 0) *lscale = (m * (1.0f / 127.0f)) * post;
}

// The next head (sequence-major index) of a walk with stride `stride` at or
// after `bh` that decodes in this launch: every head with batch-synchronous
// positions; with per-sequence positions the heads of sequences whose
// position is in [0, W) (a position >= W is recorded as an error and skipped).
// Every role of a pipeline walks the same sequence.
template <bool RAGGED>
__device__ __forceinline__ int next_decode_head(const DecodeArgs &a, int bh, int stride) {
    if constexpr (RAGGED) {
        const int BH = a.B * a.H;
        for (; bh < BH; bh += stride) {
            const int p = a.seq_pos[bh / a.H];
            if (p >= 0 && p < a.W) return bh;
            if (p >= a.W) atomicOr(&g_dev_error, kErrBadPosition);
        }
        return BH;
    } else {
        return bh;
    }
}

// The prep warps of a head (one role per warp): prep A (isA) the limbs of
// x_k = c e^L k and x_q = c e^L q and k~_t . q_t (one warp, or with NA = 2
// warp `arole` 0 x_k and warp 1 x_q and k~_t . q_t); prep-B warp `bpart` of
// NPB the new records (L_t, k~_t) and its share of the coefficient passes.
// Every token of the call is prepared before "prepared" is signalled.  With
// TC the limbs are written as the rows of the tensor-core matvec's B operand.
template <int DK, int DV, int GATE, bool BF16, bool RAGGED, int FMT, bool TC, int NA, int NPB>
__device__ __forceinline__ void prep_role(const DecodeArgs &a, const StageLayout &SL,
                                          const PrepLayout &PL, unsigned char *stages,
                                          uint64_t *full, uint64_t *prepared, uint64_t *empty,
                                          int S, bool isA, int arole, int bpart, int lane,
                                          int vblock, int vgrid, unsigned char *tiles = nullptr) {
    constexpr bool BF16S = FMT == kCodesBF16;
    const int BH = a.B * a.H, R = a.R, W = a.W, nsteps = a.n_steps;
    constexpr int CPL = DK / 32;          // contiguous key channels per lane
    const int j0 = CPL * lane;
    int i = 0;
    for (int bh = next_decode_head<RAGGED>(a, vblock, vgrid); bh < BH; bh = next_decode_head<RAGGED>(a, bh + vgrid, vgrid), ++i) {
        const int s = i % S;
        const int pos = RAGGED ? a.seq_pos[bh / a.H] : a.pos;  // records buffered
        if (!mbar_wait_bounded(&full[s], (i / S) & 1)) break;
        unsigned char *st = stages + (size_t)s * SL.bytes;
        const float *cs_s = reinterpret_cast<const float *>(st + SL.cs);
        const float *compv_s = reinterpret_cast<const float *>(st + SL.compv);
        const float *scal = reinterpret_cast<const float *>(st + SL.scal);
        float *recK_s = reinterpret_cast<float *>(st + SL.recK);
        float *recL_s = reinterpret_cast<float *>(st + SL.recL);
        const int b = bh / a.H, h = bh % a.H;
        float Ls = (GATE == 0 && pos > 0) ? recL_s[pos - 1] : 0.0f;  // scalar gate chain
        float Lc[CPL];                                             // diagonal, own channels
        if (GATE == 1 && pos > 0) {
            load_vec<CPL>(Lc, recL_s + (pos - 1) * DK + j0);
        } else {
#pragma unroll
            for (int e = 0; e < CPL; ++e) Lc[e] = 0.0f;
        }
        for (int sidx = 0; sidx < nsteps; ++sidx) {
            const int t = pos + sidx + 1, nrec = t - 1;
            const size_t tok = ((size_t)b * nsteps + sidx) * a.H + h;
            const float beta = sidx == 0 ? scal[1] : a.beta[tok];
            unsigned char *slot = st + SL.prep + sidx * PL.bytes;
            float *coefA = reinterpret_cast<float *>(slot + PL.coefA);
            float *coefG = reinterpret_cast<float *>(slot + PL.coefG);
            float g_s = 0.0f;
            if (GATE == 0) {
                Ls = Ls + logf(sidx == 0 ? scal[0] : a.alpha[tok]);
                g_s = expf(Ls);
            }
            float kj[CPL], qj[CPL], gj[CPL];
            if (sidx == 0) {
                load_io_vec<BF16, CPL>(qj, st + SL.q, j0);
                load_io_vec<BF16, CPL>(kj, st + SL.k, j0);
            } else {
                load_io_vec<BF16, CPL>(qj, a.q, tok * DK + j0);
                load_io_vec<BF16, CPL>(kj, a.k, tok * DK + j0);
            }
            if (GATE == 1) {
                float al[CPL];
                if (sidx == 0) load_vec<CPL>(al, reinterpret_cast<const float *>(st + SL.al) + j0);
                else load_vec<CPL>(al, a.alpha + tok * DK + j0);
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    Lc[e] = Lc[e] + logf(al[e]);
                    gj[e] = expf(Lc[e]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < CPL; ++e) gj[e] = g_s;
            }
            if (isA) {
                // limbs of x_k = c e^L k and x_q = c e^L q; own-token k~ . q
                int8_t *limb = reinterpret_cast<int8_t *>(slot + PL.limb);
                float *lscale = reinterpret_cast<float *>(slot + PL.lscale);
                float cj[CPL], xk[CPL], xq[CPL], kq = 0.0f;
                load_vec<CPL>(cj, cs_s + j0);
                // scalar gate with integer limbs: e^{L_t} goes into the limb
                // scales (after the split), off the split's dependency chain
                constexpr bool GPOST = GATE == 0 && !BF16S;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    const float g = GPOST ? 1.0f : gj[e];
                    xk[e] = a.delta ? cj[e] * (g * kj[e]) : 0.0f;  // b = 0 rows: no S b term
                    xq[e] = cj[e] * (g * qj[e]);
                    kq = fmaf(beta * kj[e], qj[e], kq);
                }
                const float gpost = GPOST ? g_s : 1.0f;
                // with NA = 2 prep-A warps, warp arole 0 takes x_k, warp 1 x_q and k~ . q
                const bool doK = NA == 1 || arole == 0, doQ = NA == 1 || arole == 1;
                if constexpr (BF16S) {
                    // the FP32 vectors themselves, unit scales
                    float *xs = reinterpret_cast<float *>(limb);
                    store_vec<CPL>(xs + j0, xk);
                    store_vec<CPL>(xs + DK + j0, xq);
                    if (lane == 0) lscale[0] = lscale[1] = 1.0f;
                } else {
                    // b = 0 rows: the consumers skip x_k, so it is not split
                    if constexpr (TC) {
                        // rows 8 sidx + 0..2 (x_k) and + 3..5 (x_q) of the B operand
                        int8_t *bop = reinterpret_cast<int8_t *>(tiles + (size_t)s * tc_tile_bytes(nsteps) + DV * DK);
                        if (doK && a.delta) split_limbs<CPL, 3, true>(xk, bop, DK, lscale, j0, 8 * sidx, gpost);
                        if (doQ) split_limbs<CPL, 3, true>(xq, bop, DK, lscale + 1, j0, 8 * sidx + 3, gpost);
                    } else {
                        if (a.delta) split_limbs<CPL, 3>(xk, limb, DK, lscale, j0, 0, gpost);
                        split_limbs<CPL, 3>(xq, limb, DK, lscale + 1, j0, 3, gpost);
                    }
                }
                if (doQ) {
                    kq = group_sum<32>(kq);
                    if (lane == 0) coefG[nrec + R] = kq;
                }
            } else {
                // records of this token: L_t and k~_t.  When a later token of
                // the call follows, every prep-B warp writes the same values
                // to shared memory (it reads them back there); warp 0 of them
                // also writes global memory.
                float ktj[CPL];
#pragma unroll
                for (int e = 0; e < CPL; ++e) ktj[e] = beta * kj[e];
                if (sidx + 1 < nsteps) {
                    store_vec<CPL>(recK_s + nrec * DK + j0, ktj);
                    if (GATE == 1) store_vec<CPL>(recL_s + nrec * DK + j0, Lc);
                    if (GATE == 0 && lane == 0) recL_s[nrec] = Ls;
                }
                if (bpart == 0) {
                    store_vec<CPL>(a.buf_k + ((size_t)bh * W + nrec) * DK + j0, ktj);
                    if (GATE == 1)
                        store_vec<CPL>(a.buf_gate + ((size_t)bh * W + nrec) * DK + j0, Lc);
                    if (GATE == 0 && lane == 0) a.buf_gate[(size_t)bh * W + nrec] = Ls;
                }
                __syncwarp();
                // coefficients of records 0..nrec-1 and compensators, P
                // items per pass, passes shared round-robin by the prep-B
                // warps; the 2P partial dot products of a pass are reduced
                // together with a transposing reduction
                const int nitems = nrec + R;
                float kb[CPL];  // the b-side channels: k, or 0 for the b = 0 rows
#pragma unroll
                for (int e = 0; e < CPL; ++e) kb[e] = a.delta ? kj[e] : 0.0f;
                auto coef_pass = [&](auto PC, int base) {
                    constexpr int P = decltype(PC)::value;
                    float part[2 * P];
#pragma unroll
                    for (int q8 = 0; q8 < P; ++q8) {
                        const int it = base + q8;
                        float da = 0.0f, dq = 0.0f;
                        if constexpr (GATE == 0) {
                            // scalar gate: raw dot products of the item's row
                            // (record it, or compensator it - nrec) with k and
                            // q; the gate factor is applied after the
                            // reduction.  Items past the end read the last
                            // record or compensator row and are not stored.
                            const bool isrec = it < nrec || R == 0;
                            const int ri = isrec ? min(it, nrec - 1) : min(it - nrec, R - 1);
                            const float *row = (isrec ? recK_s : compv_s) + ri * DK;
                            float w[CPL];
                            load_vec<CPL>(w, row + j0);
#pragma unroll
                            for (int e = 0; e < CPL; ++e) {
                                da = fmaf(w[e], kb[e], da);
                                dq = fmaf(w[e], qj[e], dq);
                            }
                        } else if (it < nitems) {
                            float w[CPL];
                            if (it < nrec) {
                                load_vec<CPL>(w, recK_s + it * DK + j0);
                                float Lm[CPL];
                                load_vec<CPL>(Lm, recL_s + it * DK + j0);
#pragma unroll
                                for (int e = 0; e < CPL; ++e) w[e] *= expf(Lc[e] - Lm[e]);
#pragma unroll
                                for (int e = 0; e < CPL; ++e) {
                                    da = fmaf(w[e], kb[e], da);
                                    dq = fmaf(w[e], qj[e], dq);
                                }
                            } else {
                                load_vec<CPL>(w, compv_s + (it - nrec) * DK + j0);
#pragma unroll
                                for (int e = 0; e < CPL; ++e) {
                                    da = fmaf(w[e], gj[e] * kb[e], da);
                                    dq = fmaf(w[e], gj[e] * qj[e], dq);
                                }
                            }
                        }
                        part[q8] = da;
                        part[P + q8] = dq;
                    }
                    transposed_sum<2 * P, 32>(part, lane);
                    const int idx = transposed_index<2 * P, 32>(lane);
                    const int it = base + (idx % P);
                    if (it < nitems && lane == transposed_owner<2 * P, 32>(idx)) {
                        float v = part[0];
                        // scalar gate: e^{L_t - L_m} for a record, e^{L_t} for a compensator
                        if (GATE == 0) v *= it < nrec ? expf(Ls - recL_s[it]) : g_s;
                        if (idx < P) coefA[it] = v;
                        else coefG[it] = v;
                    }
                };
                // passes of 4 items over four prep-B warps (tensor-core decode),
                // of 8 items over two (dp4a decode)
                constexpr int PI = NPB >= 4 ? 4 : 8;
                for (int base = PI * bpart; base < nitems; base += PI * NPB)
                    coef_pass(std::integral_constant<int, PI>{}, base);
            }
            __syncwarp();
        }
        // generic-proxy writes that a later asynchronous copy into this stage
        // (or the tensor-core MMA) reads or overwrites: the limbs of the MMA's
        // B operand, and the records of a multi-token call.  The coefficients
        // live in the prep slot, which no copy writes.
        if ((isA && TC) || nsteps > 1) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&prepared[s]);
            mbar_arrive(&empty[s]);
        }
    }
}

// RAGGED: per-sequence window positions (a.seq_pos); otherwise the window
// position a.pos is the same for every head and stays a kernel constant.
// FMT: the residual's storage (lq_kernels.h).
template <int DK, int DV, int GATE, bool BF16, bool RAGGED, int FMT>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeArgs a, const int S) {
    constexpr int E = BF16 ? 2 : 4;
    constexpr int RPW = DV / kConsumerWarps;  // value rows per consumer warp
    constexpr bool PACK4 = FMT == kCodesI4, BF16S = FMT == kCodesBF16;
    constexpr int CRB = code_row_bytes(FMT, DK);  // residual bytes per value row
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *prepared = full + kMaxStages;
    uint64_t *empty = prepared + kMaxStages;
    const int nsteps = a.n_steps;
    const StageLayout SL = stage_layout(DK, DV, GATE, a.R, a.pos + nsteps, nsteps, E, FMT, false, a.comp_u ? a.R : 0);
    const PrepLayout PL = prep_layout(DK, FMT);
    unsigned char *stages = smem + header_bytes();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int BH = a.B * a.H;
    const int R = a.R, W = a.W;
    const int vblock = blockIdx.x, vgrid = gridDim.x;  // this CTA's walk over the heads

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&prepared[s], kPrepWarps);
            mbar_init(&empty[s], kConsumerWarps + kPrepWarps);
        }
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    if (warp == kProducerWarp) {
        if (lane != 0) return;
        int i = 0;
        bool ok = true;
        for (int bh = next_decode_head<RAGGED>(a, vblock, vgrid); bh < BH; bh = next_decode_head<RAGGED>(a, bh + vgrid, vgrid), ++i) {
            const int s = i % S, use = i / S;
            const int pos = RAGGED ? a.seq_pos[bh / a.H] : a.pos;  // records buffered
            if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1)) {
                ok = false;
                break;
            }
            unsigned char *st = stages + (size_t)s * SL.bytes;
            const int b = bh / a.H, h = bh % a.H;
            const size_t tok = (size_t)b * nsteps * a.H + h;  // token 0 of this call
            const uint32_t in_bytes =
                nsteps > 0 ? (uint32_t)(E * (2 * DK + DV) + (GATE == 1 ? 4 * DK : 0)) : 0u;
            const uint32_t bytes = DV * CRB + 4 * DV + 4 * DK + 4 * R * DK + 4 * pos * (DK + DV) +
                                   (GATE == 1 ? 4 * pos * DK : 0) + in_bytes + (a.comp_u ? 4 * R * DV : 0);
            // small operands by 4-byte copies, tracked by the same barrier:
            // alpha and beta of token 0, the scalar-gate records, the
            // compensator rows
            float *scal = reinterpret_cast<float *>(st + SL.scal);
            if (nsteps > 0) {
                if (GATE == 0) cp_async4(scal, a.alpha + tok);
                cp_async4(scal + 1, a.beta + tok);
            }
            if (GATE == 0)
                for (int m = 0; m < pos; ++m)
                    cp_async4(st + SL.recL + 4 * m, a.buf_gate + (size_t)bh * W + m);
            for (int c = 0; c < R; ++c)
                cp_async4(st + SL.compr + 4 * c, a.comp_row + (size_t)bh * R + c);
            cp_async_mbar_arrive(&full[s]);
            mbar_arrive_expect_tx(&full[s], bytes);
            bulk_g2s(st + SL.codes, a.codes + (size_t)bh * DV * CRB, DV * CRB, &full[s]);
            bulk_g2s(st + SL.sig, a.row_scale + (size_t)bh * DV, 4 * DV, &full[s]);
            bulk_g2s(st + SL.cs, a.col_smooth + (size_t)bh * DK, 4 * DK, &full[s]);
            if (R > 0) bulk_g2s(st + SL.compv, a.comp_val + (size_t)bh * R * DK, 4 * R * DK, &full[s]);
            if (a.comp_u) bulk_g2s(st + SL.compu, a.comp_u + (size_t)bh * R * DV, 4 * R * DV, &full[s]);
            if (pos > 0) {
                bulk_g2s(st + SL.recK, a.buf_k + (size_t)bh * W * DK, 4 * pos * DK, &full[s]);
                bulk_g2s(st + SL.recU, a.buf_u + (size_t)bh * W * DV, 4 * pos * DV, &full[s]);
                if (GATE == 1)
                    bulk_g2s(st + SL.recL, a.buf_gate + (size_t)bh * W * DK, 4 * pos * DK, &full[s]);
            }
            if (nsteps > 0) {
                const unsigned char *qg = static_cast<const unsigned char *>(a.q);
                const unsigned char *kg = static_cast<const unsigned char *>(a.k);
                const unsigned char *vg = static_cast<const unsigned char *>(a.v);
                bulk_g2s(st + SL.q, qg + tok * DK * E, E * DK, &full[s]);
                bulk_g2s(st + SL.k, kg + tok * DK * E, E * DK, &full[s]);
                bulk_g2s(st + SL.v, vg + tok * DV * E, E * DV, &full[s]);
                if (GATE == 1) bulk_g2s(st + SL.al, a.alpha + tok * DK, 4 * DK, &full[s]);
            }
        }
        if (!ok) {
            // drain the copies still in flight into this CTA's shared memory
            const int issued = i;
            for (int j = issued - 1; j >= 0 && j >= issued - S; --j)
                mbar_wait_bounded(&full[j % S], (j / S) & 1);
        }
        return;
    }

    // ------------------------------------------------------------ prep warps
    if (warp >= kPrepAWarp) {
        prep_role<DK, DV, GATE, BF16, RAGGED, FMT, false, 1, kPrepBWarps>(
            a, SL, PL, stages, full, prepared, empty, S, warp == kPrepAWarp, 0, warp - kPrepBWarp, lane,
            blockIdx.x, gridDim.x);
        return;
    }

    // ------------------------------------------------------------ consumers
    constexpr int LPR16 = DK / 16, RPI16 = 32 / LPR16, NRM = RPW / RPI16;
    constexpr int LPRD = 32 / RPW;  // lanes per value row in the combine
    static_assert(NRM >= 1 && RPW % RPI16 == 0 && LPRD >= 1 && 32 % RPW == 0, "tiling");
    const int cc = lane % LPR16, sub = lane / LPR16;
    const int rloc = lane / LPRD, part = lane % LPRD;  // combine: local row, record share
    // lanes holding y_k / y_q of local row rloc after the matvec reduction
    const int src_k = (rloc % RPI16) * LPR16 + transposed_owner<2 * NRM, LPR16>(rloc / RPI16);
    const int src_q = (rloc % RPI16) * LPR16 + transposed_owner<2 * NRM, LPR16>(NRM + rloc / RPI16);

    const bool delta = a.delta != 0;  // b = 0 rows (delta = 0): no S^_0 x_k products
    int i = 0;
    for (int bh = next_decode_head<RAGGED>(a, vblock, vgrid); bh < BH; bh = next_decode_head<RAGGED>(a, bh + vgrid, vgrid), ++i) {
        const int s = i % S;
        const int pos = RAGGED ? a.seq_pos[bh / a.H] : a.pos;  // records buffered
        if (!mbar_wait_bounded(&prepared[s], (i / S) & 1)) break;
        unsigned char *st = stages + (size_t)s * SL.bytes;
        const int8_t *codes_s = reinterpret_cast<const int8_t *>(st + SL.codes);
        const float *sig_s = reinterpret_cast<const float *>(st + SL.sig);
        const int *compr_s = reinterpret_cast<const int *>(st + SL.compr);
        float *recU_s = reinterpret_cast<float *>(st + SL.recU);
        const int b = bh / a.H, h = bh % a.H;
        float *bufU = a.buf_u + (size_t)bh * W * DV;
        const int row = warp * RPW + rloc;

        for (int sidx = 0; sidx < nsteps; ++sidx) {
            const int t = pos + sidx + 1, nrec = t - 1;
            const size_t tok = ((size_t)b * nsteps + sidx) * a.H + h;
            const unsigned char *slot = st + SL.prep + sidx * PL.bytes;
            const int8_t *limb = reinterpret_cast<const int8_t *>(slot + PL.limb);
            const float *lscale = reinterpret_cast<const float *>(slot + PL.lscale);
            const float *coefA = reinterpret_cast<const float *>(slot + PL.coefA);
            const float *coefG = reinterpret_cast<const float *>(slot + PL.coefG);

            // D2: S^_0 x for this warp's rows: dp4a of the codes with the limbs.
            // A0 2^7 + A1 is exact in int32 (|.| < 2^26) and converted once;
            // the vector scales are applied after the cross-lane reduction.
            // 4-bit codes enter as 16 Q (the nibble in the high half of an
            // int8), so every sum is 16 times larger and the unit is 2^-18.
            float y;
            if constexpr (BF16S) {
                // BF16 residual: FP32 FMAs with the FP32 vectors.  Lane cc
                // takes key channels [8cc, 8cc+8) and [d_k/2 + 8cc, d_k/2 +
                // 8cc + 8), so each 16-byte read is contiguous across a row's lanes.
                const float *xs = reinterpret_cast<const float *>(limb);
                float xk[16], xq[16];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(xs + h * (DK / 2) + 8 * cc + 4 * v);
                        const float4 b4 = *reinterpret_cast<const float4 *>(xs + DK + h * (DK / 2) + 8 * cc + 4 * v);
                        const int o = 8 * h + 4 * v;
                        xk[o] = a4.x; xk[o + 1] = a4.y; xk[o + 2] = a4.z; xk[o + 3] = a4.w;
                        xq[o] = b4.x; xq[o + 1] = b4.y; xq[o + 2] = b4.z; xq[o + 3] = b4.w;
                    }
                float vals[2 * NRM];
#pragma unroll
                for (int n = 0; n < NRM; ++n) {
                    const int r = warp * RPW + n * RPI16 + sub;
                    const int8_t *rowp = codes_s + r * CRB;
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(rowp + 16 * cc);
                    const uint4 w1 = *reinterpret_cast<const uint4 *>(rowp + DK + 16 * cc);
                    const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    float ak = 0.0f, aq = 0.0f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        // element 2i in the low half of word i, 2i+1 in the high half
                        const float lo = __uint_as_float(ww[i] << 16);
                        const float hi = __uint_as_float(ww[i] & 0xFFFF0000u);
                        if (delta) {
                            ak = fmaf(lo, xk[2 * i], ak);
                            ak = fmaf(hi, xk[2 * i + 1], ak);
                        }
                        aq = fmaf(lo, xq[2 * i], aq);
                        aq = fmaf(hi, xq[2 * i + 1], aq);
                    }
                    vals[n] = ak;
                    vals[NRM + n] = aq;
                }
                transposed_sum<2 * NRM, LPR16>(vals, lane);
                y = vals[0];
            } else {
                uint4 lw[6];
#pragma unroll
                for (int v = 0; v < 6; ++v)
                    lw[v] = (v < 3 && !delta) ? make_uint4(0u, 0u, 0u, 0u)
                                              : *reinterpret_cast<const uint4 *>(limb + v * DK + 16 * cc);
                float vals[2 * NRM];
#pragma unroll
                for (int n = 0; n < NRM; ++n) {
                    const int r = warp * RPW + n * RPI16 + sub;
                    uint4 w;
                    if constexpr (PACK4) {
                        // 8 bytes = channels 16cc..16cc+15: word h holds
                        // 8h..8h+3 in its low nibbles and 8h+4..8h+7 in its high
                        const uint2 p = *reinterpret_cast<const uint2 *>(codes_s + r * CRB + 8 * cc);
                        w = make_uint4((p.x << 4) & 0xF0F0F0F0u, p.x & 0xF0F0F0F0u,
                                       (p.y << 4) & 0xF0F0F0F0u, p.y & 0xF0F0F0F0u);
                    } else {
                        w = *reinterpret_cast<const uint4 *>(codes_s + r * DK + 16 * cc);
                    }
                    int acc[6];
#pragma unroll
                    for (int v = 0; v < 6; ++v) {
                        if (v < 3 && !delta) {  // warp-uniform: the b-side sums are 0
                            acc[v] = 0;
                            continue;
                        }
                        int x = __dp4a((int)w.x, (int)lw[v].x, 0);
                        x = __dp4a((int)w.y, (int)lw[v].y, x);
                        x = __dp4a((int)w.z, (int)lw[v].z, x);
                        acc[v] = __dp4a((int)w.w, (int)lw[v].w, x);
                    }
                    // (A0 2^7 + A1) 2^7 + A2, in units of 2^-14 of the vector's scale
                    vals[n] = fmaf(__int2float_rn(acc[0] * 128 + acc[1]), 128.0f, small_int_to_f32(acc[2]));
                    vals[NRM + n] = fmaf(__int2float_rn(acc[3] * 128 + acc[4]), 128.0f, small_int_to_f32(acc[5]));
                }
                transposed_sum<2 * NRM, LPR16>(vals, lane);
                y = vals[0];
            }
            // D3-D6 for row `row`: LPRD lanes share its buffered records
            {
                const float sg = sig_s[row];
                // 2^-18 (4-bit codes enter as 16 Q), 2^-14, or 1 (FP32 sums of a BF16 residual)
                constexpr float kUnit = PACK4 ? 3.814697265625e-06f : BF16S ? 1.0f : 6.103515625e-05f;
                const float yk = delta ? __shfl_sync(0xffffffffu, y, src_k) * (sg * (lscale[0] * kUnit)) : 0.0f;
                const float yq = __shfl_sync(0xffffffffu, y, src_q) * (sg * (lscale[1] * kUnit));
                float hb = part == 0 ? yk : 0.0f, p = part == 0 ? yq : 0.0f;
                for (int m = part; m < nrec; m += LPRD) {
                    const float um = recU_s[m * DV + row];
                    hb = fmaf(coefA[m], um, hb);
                    p = fmaf(coefG[m], um, p);
                }
#pragma unroll
                for (int o = LPRD / 2; o > 0; o >>= 1) {
                    hb += __shfl_xor_sync(0xffffffffu, hb, o);
                    p += __shfl_xor_sync(0xffffffffu, p, o);
                }
                if (part == 0) {
                    if (a.comp_u) {
                        // rank-one compensators (SVD rule): u_c[row] times the coefficient
                        const float *compu_s = reinterpret_cast<const float *>(st + SL.compu);
                        for (int c = 0; c < R; ++c) {
                            const float uc = compu_s[c * DV + row];
                            hb = fmaf(coefA[nrec + c], uc, hb);
                            p = fmaf(coefG[nrec + c], uc, p);
                        }
                    } else {
                        for (int c = 0; c < R; ++c)
                            if (compr_s[c] == row) {
                                hb += coefA[nrec + c];
                                p += coefG[nrec + c];
                            }
                    }
                    const float vi = sidx == 0 ? load_io<BF16>(st + SL.v, row)
                                               : load_io<BF16>(a.v, tok * DV + row);
                    const float u = vi - hb;
                    const float o = fmaf(coefG[nrec + R], u, p);
                    store_io<BF16>(a.o, tok * DV + row, o);
                    recU_s[nrec * DV + row] = u;
                    bufU[(size_t)nrec * DV + row] = u;
                }
                __syncwarp();
            }
        }

        // release the stage to the producer
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

// ---------------------------------------------------------------------------
// Tensor-core matvec variant (d_k = d_v = 128, one int8 code per byte)
// ---------------------------------------------------------------------------
//
// The boundary matvec of D2 is a product of the 128 x 128 code matrix with
// the six limb vectors of a token (x_k limbs 0..2, x_q limbs 0..2): the
// kind::i8 tensor-core MMA computes it exactly in int32, the same sums the
// dp4a chain forms.  A kernel that allocates TMEM runs one CTA per SM, so
// the CTA holds npipe (1 or 2) independent pipelines of 12 warps, each with
// its own stage ring, barriers and TMEM columns, walking its own share of
// the heads (pipeline p of CTA c: heads c npipe + p, stride gridDim npipe);
// at most 80 registers a thread.  Roles of a pipeline (warp index mod 12):
//  * producer (warp 4, one lane): the codes by one tiled TMA box (128 rows x
//    128 bytes, 128-byte swizzle, no multicast) and the other operands by
//    bulk copies, as in decode_kernel -> "full";
//  * MMA (warp 5, one lane): 4 MMAs of 128 x N x 32 (N = 8 per token) into the
//    stage's TMEM accumulator, completion by tcgen05.commit -> "mma_done";
//  * prep A (warps 6, 7: x_k, and x_q with k~ . q) and prep B (warps 8-11,
//    records and coefficient passes): as in decode_kernel; prep A writes the
//    limbs as the rows of the MMA's K-major B operand -> "prepared";
//  * epilogue (warps 0-3): warp w reads TMEM lanes 32w..32w+31 = value rows,
//    one row per lane, so y_k and y_q arrive without any cross-lane
//    reduction; then D3-D6 for that row as in decode_kernel -> "empty".
constexpr int kTcEpiWarps = 4;
constexpr int kTcProducerWarp = 4, kTcMmaWarp = 5, kTcPrepAWarp = 6, kTcPrepAWarps = 2;
constexpr int kTcPrepBWarp = 8, kTcPrepBWarps = 4;
constexpr int kTcPrepWarps = kTcPrepAWarps + kTcPrepBWarps;
constexpr int kTcPipeWarps = 12, kTcMaxPipes = 2;
constexpr int kTcThreads = kTcMaxPipes * kTcPipeWarps * 32;
constexpr int kTcHeader = 1024;  // barriers + TMEM slot; the stages follow 1024-aligned

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// S stages per pipeline; npipe pipelines (blockDim = npipe x 12 warps);
// tcols TMEM columns allocated (S x N per pipeline).
template <int GATE, bool BF16, bool RAGGED>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const int S, const int npipe, const int tcols,
                     const __grid_constant__ CUtensorMap codes_map) {
    constexpr int DK = 128, DV = 128, FMT = kCodesI8;
    constexpr int E = BF16 ? 2 : 4;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // the swizzled operands need 1024-byte aligned addresses: align the base
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    constexpr int NBAR = kTcMaxPipes * kMaxStages;
    const int tid = threadIdx.x, lane = tid & 31;
    const int pipe = (tid >> 5) / kTcPipeWarps, warp = (tid >> 5) % kTcPipeWarps;  // role in the pipeline
    uint64_t *full = reinterpret_cast<uint64_t *>(smem) + pipe * kMaxStages;
    uint64_t *prepared = full + NBAR;
    uint64_t *mma_done = prepared + NBAR;
    uint64_t *empty = mma_done + NBAR;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint64_t *>(smem) + 4 * NBAR);
    const int nsteps = a.n_steps;
    const StageLayout SL = stage_layout(DK, DV, GATE, a.R, a.pos + nsteps, nsteps, E, FMT, true, a.comp_u ? a.R : 0);
    const PrepLayout PL = prep_layout(DK, FMT, true);
    const int TB = tc_tile_bytes(nsteps);
    // this pipeline's tiles (codes + B operand, 1024-aligned) and stages
    unsigned char *tiles = smem + kTcHeader + (size_t)pipe * S * TB;
    unsigned char *stages = smem + kTcHeader + (size_t)npipe * S * TB + (size_t)pipe * S * SL.bytes;
    const int NB = tc_rows(nsteps);  // accumulator columns per stage
    const int BH = a.B * a.H, R = a.R, W = a.W;
    const int vblock = blockIdx.x * npipe + pipe, vgrid = gridDim.x * npipe;  // this pipeline's walk

    if (tid < 32) tmem_alloc(tmem_slot, tcols);
    if (tid == 0) {
        uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
        for (int q = 0; q < npipe; ++q)
            for (int s = 0; s < S; ++s) {
                mbar_init(&bars[q * kMaxStages + s], 1);                                // full
                mbar_init(&bars[NBAR + q * kMaxStages + s], kTcPrepWarps);             // prepared
                mbar_init(&bars[2 * NBAR + q * kMaxStages + s], 1);                    // mma_done
                mbar_init(&bars[3 * NBAR + q * kMaxStages + s], kTcEpiWarps + kTcPrepWarps);  // empty
            }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot + (uint32_t)(pipe * S * NB);  // this pipeline's columns

    if (warp == kTcProducerWarp) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int i = 0;
            bool ok = true;
            for (int bh = next_decode_head<RAGGED>(a, vblock, vgrid); bh < BH;
                 bh = next_decode_head<RAGGED>(a, bh + vgrid, vgrid), ++i) {
                const int s = i % S, use = i / S;
                const int pos = RAGGED ? a.seq_pos[bh / a.H] : a.pos;  // records buffered
                if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1)) {
                    ok = false;
                    break;
                }
                unsigned char *st = stages + (size_t)s * SL.bytes;
                const int b = bh / a.H, h = bh % a.H;
                const size_t tok = (size_t)b * nsteps * a.H + h;  // token 0 of this call
                const uint32_t in_bytes = (uint32_t)(E * (2 * DK + DV) + (GATE == 1 ? 4 * DK : 0));
                const uint32_t bytes = DV * DK + 4 * DV + 4 * DK + 4 * R * DK + 4 * pos * (DK + DV) +
                                       (GATE == 1 ? 4 * pos * DK : 0) + in_bytes + (a.comp_u ? 4 * R * DV : 0);
                float *scal = reinterpret_cast<float *>(st + SL.scal);
                if (GATE == 0) cp_async4(scal, a.alpha + tok);
                cp_async4(scal + 1, a.beta + tok);
                if (GATE == 0)
                    for (int m = 0; m < pos; ++m)
                        cp_async4(st + SL.recL + 4 * m, a.buf_gate + (size_t)bh * W + m);
                for (int c = 0; c < R; ++c)
                    cp_async4(st + SL.compr + 4 * c, a.comp_row + (size_t)bh * R + c);
                cp_async_mbar_arrive(&full[s]);
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(tiles + (size_t)s * TB, &codes_map, 0, bh * DV, &full[s]);
                bulk_g2s(st + SL.sig, a.row_scale + (size_t)bh * DV, 4 * DV, &full[s]);
                bulk_g2s(st + SL.cs, a.col_smooth + (size_t)bh * DK, 4 * DK, &full[s]);
                if (R > 0) bulk_g2s(st + SL.compv, a.comp_val + (size_t)bh * R * DK, 4 * R * DK, &full[s]);
                if (a.comp_u) bulk_g2s(st + SL.compu, a.comp_u + (size_t)bh * R * DV, 4 * R * DV, &full[s]);
                if (pos > 0) {
                    bulk_g2s(st + SL.recK, a.buf_k + (size_t)bh * W * DK, 4 * pos * DK, &full[s]);
                    bulk_g2s(st + SL.recU, a.buf_u + (size_t)bh * W * DV, 4 * pos * DV, &full[s]);
                    if (GATE == 1)
                        bulk_g2s(st + SL.recL, a.buf_gate + (size_t)bh * W * DK, 4 * pos * DK, &full[s]);
                }
                const unsigned char *qg = static_cast<const unsigned char *>(a.q);
                const unsigned char *kg = static_cast<const unsigned char *>(a.k);
                const unsigned char *vg = static_cast<const unsigned char *>(a.v);
                bulk_g2s(st + SL.q, qg + tok * DK * E, E * DK, &full[s]);
                bulk_g2s(st + SL.k, kg + tok * DK * E, E * DK, &full[s]);
                bulk_g2s(st + SL.v, vg + tok * DV * E, E * DV, &full[s]);
                if (GATE == 1) bulk_g2s(st + SL.al, a.alpha + tok * DK, 4 * DK, &full[s]);
            }
            if (!ok) {
                // drain the copies still in flight into this CTA's shared memory
                for (int j = i - 1; j >= 0 && j >= i - S; --j) mbar_wait_bounded(&full[j % S], (j / S) & 1);
            }
        }
    } else if (warp >= kTcPrepAWarp) {
        // ---------------------------------------------------------- prep
        prep_role<DK, DV, GATE, BF16, RAGGED, FMT, true, kTcPrepAWarps, kTcPrepBWarps>(
            a, SL, PL, stages, full, prepared, empty, S, warp < kTcPrepBWarp, warp - kTcPrepAWarp,
            warp - kTcPrepBWarp, lane, vblock, vgrid, tiles);
    } else if (warp == kTcMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(DV, NB);
            int i = 0, last = -1;
            for (int bh = next_decode_head<RAGGED>(a, vblock, vgrid); bh < BH;
                 bh = next_decode_head<RAGGED>(a, bh + vgrid, vgrid), ++i) {
                const int s = i % S;
                if (!mbar_wait_bounded(&full[s], (i / S) & 1)) break;
                if (!mbar_wait_bounded(&prepared[s], (i / S) & 1)) break;
                tc_fence_after_sync();
                const uint32_t a0 = smem_u32(tiles + (size_t)s * TB), b0 = a0 + DV * DK;
#pragma unroll
                for (int k = 0; k < DK / 32; ++k)
                    mma_i8(tmem + (uint32_t)(s * NB), smem_desc_sw128(a0 + 32 * k),
                           smem_desc_sw128(b0 + 32 * k), idesc, k > 0);
                mma_commit(&mma_done[s]);
                last = i;
            }
            // every MMA issued has completed before TMEM is released
            if (last >= 0) mbar_wait_bounded(&mma_done[last % S], (last / S) & 1);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int row = warp * 32 + lane;  // TMEM lane = value row
        const uint32_t tlane = (uint32_t)(warp * 32) << 16;
        const bool delta = a.delta != 0;
        int i = 0;
        for (int bh = next_decode_head<RAGGED>(a, vblock, vgrid); bh < BH;
             bh = next_decode_head<RAGGED>(a, bh + vgrid, vgrid), ++i) {
            const int s = i % S;
            const int pos = RAGGED ? a.seq_pos[bh / a.H] : a.pos;  // records buffered
            if (!mbar_wait_bounded(&mma_done[s], (i / S) & 1)) break;
            if (!mbar_wait_bounded(&prepared[s], (i / S) & 1)) break;
            tc_fence_after_sync();
            unsigned char *st = stages + (size_t)s * SL.bytes;
            const float *sig_s = reinterpret_cast<const float *>(st + SL.sig);
            const int *compr_s = reinterpret_cast<const int *>(st + SL.compr);
            float *recU_s = reinterpret_cast<float *>(st + SL.recU);
            const int b = bh / a.H, h = bh % a.H;
            float *bufU = a.buf_u + (size_t)bh * W * DV;
            const float sg = sig_s[row];
            for (int sidx = 0; sidx < nsteps; ++sidx) {
                const int t = pos + sidx + 1, nrec = t - 1;
                const size_t tok = ((size_t)b * nsteps + sidx) * a.H + h;
                const unsigned char *slot = st + SL.prep + sidx * PL.bytes;
                const float *lscale = reinterpret_cast<const float *>(slot + PL.lscale);
                const float *coefA = reinterpret_cast<const float *>(slot + PL.coefA);
                const float *coefG = reinterpret_cast<const float *>(slot + PL.coefG);
                // D2: the six exact int32 limb sums of this row; (A0 2^7 + A1)
                // 2^7 + A2 in units of 2^-14 of the vector's scale
                int acc[8];
                tmem_load8_i32(tmem + tlane + (uint32_t)(s * NB + 8 * sidx), acc);
                const float vk = fmaf(__int2float_rn(acc[0] * 128 + acc[1]), 128.0f, small_int_to_f32(acc[2]));
                const float vq = fmaf(__int2float_rn(acc[3] * 128 + acc[4]), 128.0f, small_int_to_f32(acc[5]));
                constexpr float kUnit = 6.103515625e-05f;  // 2^-14
                // D3-D6 for this row
                float hb = delta ? vk * (sg * (lscale[0] * kUnit)) : 0.0f;
                float p = vq * (sg * (lscale[1] * kUnit));
                int m = 0;
                for (; m + 4 <= nrec; m += 4) {  // coefficients are 16-byte aligned
                    const float4 ca = *reinterpret_cast<const float4 *>(coefA + m);
                    const float4 cg = *reinterpret_cast<const float4 *>(coefG + m);
                    const float u0 = recU_s[m * DV + row], u1 = recU_s[(m + 1) * DV + row];
                    const float u2 = recU_s[(m + 2) * DV + row], u3 = recU_s[(m + 3) * DV + row];
                    hb = fmaf(ca.x, u0, hb);
                    p = fmaf(cg.x, u0, p);
                    hb = fmaf(ca.y, u1, hb);
                    p = fmaf(cg.y, u1, p);
                    hb = fmaf(ca.z, u2, hb);
                    p = fmaf(cg.z, u2, p);
                    hb = fmaf(ca.w, u3, hb);
                    p = fmaf(cg.w, u3, p);
                }
                for (; m < nrec; ++m) {
                    const float um = recU_s[m * DV + row];
                    hb = fmaf(coefA[m], um, hb);
                    p = fmaf(coefG[m], um, p);
                }
                if (a.comp_u) {
                    // rank-one compensators (SVD rule): u_c[row] times the coefficient
                    const float *compu_s = reinterpret_cast<const float *>(st + SL.compu);
                    for (int c = 0; c < R; ++c) {
                        const float uc = compu_s[c * DV + row];
                        hb = fmaf(coefA[nrec + c], uc, hb);
                        p = fmaf(coefG[nrec + c], uc, p);
                    }
                } else {
                    for (int c = 0; c < R; ++c)
                        if (compr_s[c] == row) {
                            hb += coefA[nrec + c];
                            p += coefG[nrec + c];
                        }
                }
                const float vi = sidx == 0 ? load_io<BF16>(st + SL.v, row) : load_io<BF16>(a.v, tok * DV + row);
                const float u = vi - hb;
                const float o = fmaf(coefG[nrec + R], u, p);
                store_io<BF16>(a.o, tok * DV + row, o);
                recU_s[nrec * DV + row] = u;
                bufU[(size_t)nrec * DV + row] = u;
            }
            // this head's TMEM reads are complete: release the stage (and its
            // accumulator) to the producer
            tc_fence_before_sync();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (tid < 32) {
        tc_fence_after_sync();
        tmem_dealloc(*tmem_slot, tcols);
    }
}

// The 2-D map of all codes [B*H*128 rows][128 bytes]: one box = one head's
// 128 x 128 codes, stored with the 128-byte swizzle.
bool codes_tensor_map(CUtensorMap *m, const int8_t *codes, long long rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, 128};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(codes), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int GATE, bool BF16, bool RAGGED>
cudaError_t launch_tc(const DecodeArgs &a, cudaStream_t stream) {
    constexpr int E = BF16 ? 2 : 4;
    static std::atomic<uint64_t> configured{0};  // devices already set up
    static int sm_count[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = decode_tc_kernel<GATE, BF16, RAGGED>;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        int optin = 0, sms = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        sm_count[dev & 63] = sms;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const StageLayout SL = stage_layout(128, 128, GATE, a.R, a.pos + a.n_steps, a.n_steps, E, kCodesI8, true,
                                        a.comp_u ? a.R : 0);
    const int fixed = 1024 + kTcHeader;  // alignment slack + header
    const int NB = tc_rows(a.n_steps);
    const int per_stage = SL.bytes + tc_tile_bytes(a.n_steps);
    auto cols_for = [NB](int cols) {
        int c = 32;
        while (c < cols) c <<= 1;
        return c;
    };
    // one CTA per SM; two pipelines when each gets at least two stages,
    // else one pipeline with as many stages as fit (shared memory and the
    // 512 TMEM columns)
    const int per_sm = 227 * 1024;  // the one CTA of the SM takes all of it
    int npipe = 2, S = (per_sm - fixed) / (2 * per_stage);
    if (S > kMaxStages) S = kMaxStages;
    while (S >= 2 && cols_for(2 * S * NB) > 512) --S;
    if (S < 2) {
        npipe = 1;
        S = (per_sm - fixed) / per_stage;
        if (S > kMaxStages) S = kMaxStages;
        while (S >= 1 && cols_for(S * NB) > 512) --S;
    }
    if (S < 1) return cudaErrorInvalidConfiguration;
    const int smem = fixed + npipe * S * per_stage;
    CUtensorMap map;
    if (!codes_tensor_map(&map, a.codes, (long long)a.B * a.H * 128)) return cudaErrorInvalidValue;
    const int BH = a.B * a.H;
    int grid = sm_count[dev & 63];
    if (grid * npipe > BH) grid = (BH + npipe - 1) / npipe;
    kern<<<grid, npipe * kTcPipeWarps * 32, smem, stream>>>(a, S, npipe, cols_for(npipe * S * NB), map);
    return cudaGetLastError();
}

template <int DK, int DV, int GATE, bool BF16, bool RAGGED, int FMT>
cudaError_t launch_d(const DecodeArgs &a, cudaStream_t stream) {
    constexpr int E = BF16 ? 2 : 4;
    static std::atomic<uint64_t> configured{0};  // devices already set up
    static int sm_count[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = decode_kernel<DK, DV, GATE, BF16, RAGGED, FMT>;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        int optin = 0, sms = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        sm_count[dev & 63] = sms;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    // a stage holds the records this launch reads and writes (pos + n_steps)
    const StageLayout SL = stage_layout(DK, DV, GATE, a.R, a.pos + a.n_steps, a.n_steps, E, FMT, false,
                                        a.comp_u ? a.R : 0);
    const int fixed = header_bytes();
    // two CTAs per SM when registers allow it and each can hold at least
    // two stages, else one CTA per SM with as many stages as fit
    const int per_sm = 227 * 1024;
    int ctas = 2, S = (per_sm / 2 - 1024 - fixed) / SL.bytes;
    if (S > kMaxStages) S = kMaxStages;
    int smem = fixed + S * SL.bytes;
    int resident = 0;
    if (S >= 2) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, kThreads, smem);
        if (e != cudaSuccess) return e;
    }
    if (S < 2 || resident < 2) {
        ctas = 1;
        S = (per_sm - 1024 - fixed) / SL.bytes;
        if (S > kMaxStages) S = kMaxStages;
        smem = fixed + S * SL.bytes;
    }
    if (S < 1) return cudaErrorInvalidConfiguration;
    const int BH = a.B * a.H;
    int grid = sm_count[dev & 63] * ctas;
    if (grid > BH) grid = BH;
    kern<<<grid, kThreads, smem, stream>>>(a, S);
    return cudaGetLastError();
}

template <int DK, int DV, int GATE, bool BF16>
cudaError_t launch_dr(const DecodeArgs &a, cudaStream_t stream) {
    const int fmt = code_format(a.bits);
    if constexpr (DK == 128 && DV == 128) {
        if (fmt == kCodesI8)  // the tensor-core matvec
            return a.seq_pos ? launch_tc<GATE, BF16, true>(a, stream) : launch_tc<GATE, BF16, false>(a, stream);
    }
    if (fmt == kCodesI4)
        return a.seq_pos ? launch_d<DK, DV, GATE, BF16, true, kCodesI4>(a, stream)
                         : launch_d<DK, DV, GATE, BF16, false, kCodesI4>(a, stream);
    if (fmt == kCodesBF16)
        return a.seq_pos ? launch_d<DK, DV, GATE, BF16, true, kCodesBF16>(a, stream)
                         : launch_d<DK, DV, GATE, BF16, false, kCodesBF16>(a, stream);
    return a.seq_pos ? launch_d<DK, DV, GATE, BF16, true, kCodesI8>(a, stream)
                     : launch_d<DK, DV, GATE, BF16, false, kCodesI8>(a, stream);
}

template <int DK, int DV>
cudaError_t launch_decode_d(const DecodeArgs &a, int gate, bool bf16, cudaStream_t stream) {
    if (gate == 1)
        return bf16 ? launch_dr<DK, DV, 1, true>(a, stream) : launch_dr<DK, DV, 1, false>(a, stream);
    return bf16 ? launch_dr<DK, DV, 0, true>(a, stream) : launch_dr<DK, DV, 0, false>(a, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, int d_k, int d_v, int gate, bool bf16,
                          cudaStream_t stream) {
    if (a.n_steps < 1) return cudaErrorInvalidValue;
    if (a.bits != 8 && a.bits != 6 && a.bits != 4 && a.bits != 16) return cudaErrorInvalidValue;
    if (d_k == 128 && d_v == 128) return launch_decode_d<128, 128>(a, gate, bf16, stream);
    if (d_k == 128 && d_v == 64) return launch_decode_d<128, 64>(a, gate, bf16, stream);
    if (d_k == 64 && d_v == 128) return launch_decode_d<64, 128>(a, gate, bf16, stream);
    if (d_k == 64 && d_v == 64) return launch_decode_d<64, 64>(a, gate, bf16, stream);
    return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_dev_error(unsigned int *out) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_dev_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(unsigned int));
}

}  // namespace lq
