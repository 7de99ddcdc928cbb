// lq_decode.cu -- per-window int8 decode (and window commit) on sm_100a.
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
// of real tokens), so they enter with decay e^{L_t}.
//
// Kernel structure (persistent, warp-specialised):
//  * a grid of at most (SMs x CTAs per SM) CTAs walks the (sequence, head)
//    pairs with a grid stride;
//  * warp 8 of each CTA is the producer: one lane streams every head's int8
//    codes, scales, smoothing factors, compensators, buffered records and the
//    token's q/k/v into a ring of shared-memory stages with 1-D bulk copies
//    (no multicast), one "full" mbarrier per stage;
//  * warps 0-7 consume: the codes are dequantized in registers and multiplied
//    against two vectors at once (FP32 FMA), the two dot products of each row
//    are reduced with a transposing warp reduction, then each value channel
//    forms u_t and o_t.  The next head's scalar inputs are prefetched into
//    registers while the current head is computed.  Consumers synchronise on
//    named barrier 1 and release a stage through its "empty" mbarrier;
//  * when the window fills (or for a standalone commit, launched with no
//    tokens) the consumers rebuild the FP32 state of the head in registers and
//    re-quantize it in place (lq_quant.cuh).
// Every wait is bounded (lq_common.cuh); a wait that expires sets the device
// error word and the CTA stops consuming.
#include <atomic>
#include <cstddef>

#include "lq_kernels.h"
#include "lq_quant.cuh"

namespace lq {

__device__ unsigned int g_dev_error = 0;

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxStages = 8;
constexpr int kCoef = 32 + kMaxComp + 1;

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }

// Byte offsets inside one stage (one head's operands).
struct StageLayout {
    int codes, sig, cs, compv, compr, recK, recU, recL, q, k, v, al, bytes;
};

__host__ __device__ inline StageLayout stage_layout(int DK, int DV, int gate, int R, int W, int e) {
    StageLayout L{};
    int o = 0;
    L.codes = o; o += align16(DV * DK);
    L.sig = o;   o += align16(4 * DV);
    L.cs = o;    o += align16(4 * DK);
    L.compv = o; o += align16(4 * R * DK);
    L.compr = o; o += align16(4 * kMaxComp);
    L.recK = o;  o += align16(4 * W * DK);
    L.recU = o;  o += align16(4 * W * DV);
    L.recL = o;  o += align16(4 * W * (gate == 1 ? DK : 1));
    L.q = o;     o += align16(e * DK);
    L.k = o;     o += align16(e * DK);
    L.v = o;     o += align16(e * DV);
    L.al = o;    o += gate == 1 ? align16(4 * DK) : 0;
    L.bytes = align16(o);
    return L;
}

// Per-CTA scratch shared by the consumer warps.  Members read with 16-byte
// vector loads (xk, xq, and the quantizer's colpart) are 16-byte aligned; the
// scratch itself starts on a 16-byte boundary after the stages.
template <int DK, int DV>
struct alignas(16) Scratch {
    alignas(16) float qf[DK];
    alignas(16) float kf[DK];
    alignas(16) float gk[DK];
    alignas(16) float gq[DK];
    alignas(16) float xk[DK];
    alignas(16) float xq[DK];
    alignas(16) float kt[DK];
    // x_k and x_q split into three int8 limbs per 16-column chunk:
    // x ~= s_chunk * (X0 + X1 / 2^7 + X2 / 2^14)
    alignas(16) int8_t limb[6][DK];
    float lscale[2][DK / 16];
    float coefA[kCoef], coefG[kCoef];
    float y[2 * DV];
    float misc[4];
    QuantSmem<DK, DV, kConsumerWarps> quant;
};
using ScratchA = Scratch<128, 128>;
using ScratchB = Scratch<64, 64>;
using ScratchC = Scratch<64, 128>;
using QuantA = QuantSmem<128, 128, kConsumerWarps>;
using QuantB = QuantSmem<64, 64, kConsumerWarps>;
static_assert(offsetof(ScratchA, xk) % 16 == 0 && offsetof(ScratchB, xq) % 16 == 0 &&
                  offsetof(ScratchA, quant) % 16 == 0 && offsetof(ScratchC, quant) % 16 == 0 &&
                  offsetof(QuantA, colpart) % 16 == 0 && offsetof(QuantB, colpart) % 16 == 0,
              "vector-accessed scratch must be 16-byte aligned");

__host__ __device__ constexpr int header_bytes() { return 2 * kMaxStages * 8; }

// Splits x_j (held by thread j of a 16-thread chunk) into three int8 limbs
// with a per-chunk scale s = max|x| / 127:  x ~= s (X0 + X1/2^7 + X2/2^14),
// |error| <= s / 2^15.  Writes limb[0..2][j] and lscale[j / 16].
template <int DKL>
__device__ __forceinline__ void split_limbs_t(float x, int8_t (*limb)[DKL], float *lscale, int j) {
    float m = fabsf(x);
#pragma unroll
    for (int s = 8; s > 0; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
    const float inv = m > 0.0f ? __fdiv_rn(127.0f, m) : 0.0f;
    const float t = x * inv;
    const float x0 = rintf(t);
    const float r1 = (t - x0) * 128.0f;
    const float x1 = rintf(r1);
    const float x2 = rintf((r1 - x1) * 128.0f);
    limb[0][j] = (int8_t)(int)x0;
    limb[1][j] = (int8_t)(int)x1;
    limb[2][j] = (int8_t)(int)x2;
    if ((j & 15) == 0) lscale[j >> 4] = m * (1.0f / 127.0f);
}

template <int DK, int DV, int GATE, bool BF16, bool COMMIT>
__global__ void __launch_bounds__(kThreads, COMMIT ? 1 : 2) decode_kernel(const DecodeArgs a, const int S) {
    using T = Tile<DK, DV, kConsumerWarps>;
    constexpr int E = BF16 ? 2 : 4;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kMaxStages;
    const StageLayout SL = stage_layout(DK, DV, GATE, a.R, a.W, E);
    unsigned char *stages = smem + header_bytes();
    auto &sc = *reinterpret_cast<Scratch<DK, DV> *>(stages + (size_t)S * SL.bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int BH = a.B * a.H;
    const int R = a.R, W = a.W, pos = a.pos, nsteps = a.n_steps;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    if (warp == kConsumerWarps) {
        if (lane != 0) return;
        int i = 0;
        bool ok = true;
        for (int bh = blockIdx.x; bh < BH; bh += gridDim.x, ++i) {
            const int s = i % S, use = i / S;
            if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1)) {
                ok = false;
                break;
            }
            unsigned char *st = stages + (size_t)s * SL.bytes;
            const int b = bh / a.H, h = bh % a.H;
            const size_t tok = (size_t)b * nsteps * a.H + h;  // token 0 of this call
            const uint32_t in_bytes =
                nsteps > 0 ? (uint32_t)(E * (2 * DK + DV) + (GATE == 1 ? 4 * DK : 0)) : 0u;
            const uint32_t bytes = DV * DK + 4 * DV + 4 * DK + 4 * R * DK + 4 * pos * (DK + DV) +
                                   (GATE == 1 ? 4 * pos * DK : 0) + in_bytes;
            mbar_arrive_expect_tx(&full[s], bytes);
            bulk_g2s(st + SL.codes, a.codes + (size_t)bh * DV * DK, DV * DK, &full[s]);
            bulk_g2s(st + SL.sig, a.row_scale + (size_t)bh * DV, 4 * DV, &full[s]);
            bulk_g2s(st + SL.cs, a.col_smooth + (size_t)bh * DK, 4 * DK, &full[s]);
            if (R > 0) bulk_g2s(st + SL.compv, a.comp_val + (size_t)bh * R * DK, 4 * R * DK, &full[s]);
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

    // ------------------------------------------------------------ consumers
    const int c0 = T::col0(lane);
    // registers prefetched one head ahead: scalar gate and beta of token 0,
    // the last scalar-gate record L_pos (every thread), the scalar-gate
    // records (thread m holds L_{m+1}) and the compensator rows
    float pf_alpha = 0.f, pf_beta = 0.f, pf_L = 0.f, pf_Lprev = 0.f;
    int pf_comp = 0;
    auto prefetch = [&](int bh) {
        if (bh >= BH) return;
        const int b = bh / a.H, h = bh % a.H;
        const size_t tok = (size_t)b * nsteps * a.H + h;
        if (nsteps > 0) {
            if (GATE == 0) pf_alpha = a.alpha[tok];
            pf_beta = a.beta[tok];
        }
        if (GATE == 0 && pos > 0) pf_Lprev = a.buf_gate[(size_t)bh * W + pos - 1];
        if (GATE == 0 && tid < pos) pf_L = a.buf_gate[(size_t)bh * W + tid];
        if (tid < R) pf_comp = a.comp_row[(size_t)bh * R + tid];
    };
    prefetch(blockIdx.x);

    int i = 0;
    for (int bh = blockIdx.x; bh < BH; bh += gridDim.x, ++i) {
        const int s = i % S;
        const float cur_alpha = pf_alpha, cur_beta = pf_beta, cur_L = pf_L, cur_Lprev = pf_Lprev;
        const int cur_comp = pf_comp;
        prefetch(bh + gridDim.x);
        const bool ok = mbar_wait_bounded(&full[s], (i / S) & 1);

        unsigned char *st = stages + (size_t)s * SL.bytes;
        const int8_t *codes_s = reinterpret_cast<const int8_t *>(st + SL.codes);
        const float *sig_s = reinterpret_cast<const float *>(st + SL.sig);
        const float *cs_s = reinterpret_cast<const float *>(st + SL.cs);
        const float *compv_s = reinterpret_cast<const float *>(st + SL.compv);
        float *recK_s = reinterpret_cast<float *>(st + SL.recK);
        float *recU_s = reinterpret_cast<float *>(st + SL.recU);
        float *recL_s = reinterpret_cast<float *>(st + SL.recL);
        int *compr_s = reinterpret_cast<int *>(st + SL.compr);
        const int b = bh / a.H, h = bh % a.H;
        float *bufL = a.buf_gate + (size_t)bh * W * (GATE == 1 ? DK : 1);
        float *bufK = a.buf_k + (size_t)bh * W * DK;
        float *bufU = a.buf_u + (size_t)bh * W * DV;
        if (GATE == 0 && tid < pos) recL_s[tid] = cur_L;
        if (tid < R) compr_s[tid] = cur_comp;

        bool abort = false;
        for (int sidx = 0; sidx < nsteps; ++sidx) {
            const int t = pos + sidx + 1;
            const size_t tok = ((size_t)b * nsteps + sidx) * a.H + h;
            const float beta = sidx == 0 ? cur_beta : a.beta[tok];
            float vi = 0.f;
            // D1: inputs, running log gate, k~
            if (tid < DK) {
                float qj, kj, al;
                if (sidx == 0) {
                    qj = load_io<BF16>(st + SL.q, tid);
                    kj = load_io<BF16>(st + SL.k, tid);
                    al = GATE == 1 ? reinterpret_cast<const float *>(st + SL.al)[tid] : cur_alpha;
                } else {
                    qj = load_io<BF16>(a.q, tok * DK + tid);
                    kj = load_io<BF16>(a.k, tok * DK + tid);
                    al = GATE == 1 ? a.alpha[tok * DK + tid] : a.alpha[tok];
                }
                float Lt;
                if (GATE == 1) {
                    const float prev = t > 1 ? recL_s[(t - 2) * DK + tid] : 0.0f;
                    Lt = prev + logf(al);
                    recL_s[(t - 1) * DK + tid] = Lt;
                    bufL[(size_t)(t - 1) * DK + tid] = Lt;
                } else {
                    // L_{t-1}: the prefetched register for the first token,
                    // else the record thread 0 wrote one token earlier
                    const float prev = sidx == 0 ? (t > 1 ? cur_Lprev : 0.0f) : recL_s[t - 2];
                    Lt = prev + logf(al);
                    if (tid == 0) {
                        sc.misc[0] = Lt;
                        recL_s[t - 1] = Lt;
                        bufL[t - 1] = Lt;
                    }
                }
                const float g = expf(Lt);
                const float ktj = beta * kj;
                sc.qf[tid] = qj;
                sc.kf[tid] = kj;
                sc.gk[tid] = g * kj;
                sc.gq[tid] = g * qj;
                const float xk = cs_s[tid] * (g * kj), xq = cs_s[tid] * (g * qj);
                sc.xk[tid] = xk;
                sc.xq[tid] = xq;
                sc.kt[tid] = ktj;
                split_limbs_t<DK>(xk, &sc.limb[0], sc.lscale[0], tid);
                split_limbs_t<DK>(xq, &sc.limb[3], sc.lscale[1], tid);
                recK_s[(t - 1) * DK + tid] = ktj;
                bufK[(size_t)(t - 1) * DK + tid] = ktj;
            }
            if (tid < DV) vi = sidx == 0 ? load_io<BF16>(st + SL.v, tid) : load_io<BF16>(a.v, tok * DV + tid);
            if (sidx == 0) {
                if (consumer_sync_or<kConsumers>(!ok)) {
                    abort = true;
                    break;
                }
            } else {
                consumer_sync<kConsumers>();
            }

            // D3 coefficients: records 1..t-1, compensators, own token.  Each
            // warp takes up to four items per pass; the eight partial dot
            // products are reduced together with a transposing reduction.
            {
                const float Lt_s = GATE == 0 ? sc.misc[0] : 0.0f;
                const int nrec = t - 1, nitems = nrec + R + 1;
                for (int base = warp * 4; base < nitems; base += kConsumerWarps * 4) {
                    float part[8];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int it = base + q4;
                        float da = 0.0f, dq = 0.0f;
                        if (it < nrec) {
                            const float *km = recK_s + it * DK;
                            if (GATE == 1) {
                                const float *Lm = recL_s + it * DK;
                                const float *Lt = recL_s + (t - 1) * DK;
#pragma unroll
                                for (int e = 0; e < DK / 32; ++e) {
                                    const int j = lane + 32 * e;
                                    const float w = km[j] * expf(Lt[j] - Lm[j]);
                                    da = fmaf(w, sc.kf[j], da);
                                    dq = fmaf(w, sc.qf[j], dq);
                                }
                            } else {
#pragma unroll
                                for (int e = 0; e < DK / 32; ++e) {
                                    const int j = lane + 32 * e;
                                    da = fmaf(km[j], sc.kf[j], da);
                                    dq = fmaf(km[j], sc.qf[j], dq);
                                }
                            }
                        } else if (it < nrec + R) {
                            const float *cv = compv_s + (it - nrec) * DK;
#pragma unroll
                            for (int e = 0; e < DK / 32; ++e) {
                                const int j = lane + 32 * e;
                                da = fmaf(cv[j], sc.gk[j], da);
                                dq = fmaf(cv[j], sc.gq[j], dq);
                            }
                        } else if (it == nrec + R) {
#pragma unroll
                            for (int e = 0; e < DK / 32; ++e) {
                                const int j = lane + 32 * e;
                                dq = fmaf(sc.kt[j], sc.qf[j], dq);
                            }
                        }
                        part[q4] = da;
                        part[4 + q4] = dq;
                    }
                    transposed_sum<8, 32>(part, lane);
                    const int idx = transposed_index<8, 32>(lane);
                    const int it = base + (idx & 3);
                    if (it < nitems && lane == transposed_owner<8, 32>(idx)) {
                        float v = part[0];
                        if (GATE == 0 && it < nrec) v *= expf(Lt_s - recL_s[it]);
                        if (idx < 4) sc.coefA[it] = v;
                        else sc.coefG[it] = v;
                    }
                }
            }

            // D2: y_k = Q (c e^L k), y_q = Q (c e^L q): integer dot products of
            // the int8 codes with the int8 limbs of both vectors (dp4a), one
            // 16-code chunk per lane, combined per chunk in FP32 and reduced
            // across the row's lanes with a transposing reduction
            {
                constexpr int LPR16 = DK / 16, RPI16 = 32 / LPR16, RPW = DV / kConsumerWarps;
                constexpr int NRM = RPW / RPI16;
                static_assert(NRM >= 1 && RPW % RPI16 == 0, "matvec tiling");
                const int cc = lane % LPR16, sub = lane / LPR16;
                uint4 lw[6];
#pragma unroll
                for (int v = 0; v < 6; ++v) lw[v] = *reinterpret_cast<const uint4 *>(&sc.limb[v][16 * cc]);
                int acc[NRM][6];
#pragma unroll
                for (int n = 0; n < NRM; ++n) {
                    const int row = warp * RPW + n * RPI16 + sub;
                    const uint4 w = *reinterpret_cast<const uint4 *>(codes_s + row * DK + 16 * cc);
#pragma unroll
                    for (int v = 0; v < 6; ++v) {
                        int x = __dp4a((int)w.x, (int)lw[v].x, 0);
                        x = __dp4a((int)w.y, (int)lw[v].y, x);
                        x = __dp4a((int)w.z, (int)lw[v].z, x);
                        acc[n][v] = __dp4a((int)w.w, (int)lw[v].w, x);
                    }
                }
                const float sk = sc.lscale[0][cc], sq = sc.lscale[1][cc];
                float vals[2 * NRM];
#pragma unroll
                for (int n = 0; n < NRM; ++n) {
                    vals[n] = sk * fmaf((float)acc[n][2], 6.103515625e-05f,
                                        fmaf((float)acc[n][1], 0.0078125f, (float)acc[n][0]));
                    vals[NRM + n] = sq * fmaf((float)acc[n][5], 6.103515625e-05f,
                                              fmaf((float)acc[n][4], 0.0078125f, (float)acc[n][3]));
                }
                transposed_sum<2 * NRM, LPR16>(vals, lane);
                const int idx = transposed_index<2 * NRM, LPR16>(lane);
                const int row = warp * RPW + (idx % NRM) * RPI16 + sub;
                sc.y[(idx / NRM) * DV + row] = vals[0] * sig_s[row];
            }
            consumer_sync<kConsumers>();

            // D3-D6 per value channel: correction, u_t, o_t, record
            if (tid < DV) {
                const int nrec = t - 1;
                float hb = sc.y[tid], p = sc.y[DV + tid];
                for (int c = 0; c < R; ++c)
                    if (compr_s[c] == tid) {
                        hb += sc.coefA[nrec + c];
                        p += sc.coefG[nrec + c];
                    }
                for (int m = 0; m < nrec; ++m) {
                    const float um = recU_s[m * DV + tid];
                    hb = fmaf(sc.coefA[m], um, hb);
                    p = fmaf(sc.coefG[m], um, p);
                }
                const float u = vi - hb;
                const float o = fmaf(sc.coefG[nrec + R], u, p);
                store_io<BF16>(a.o, tok * DV + tid, o);
                recU_s[(t - 1) * DV + tid] = u;
                bufU[(size_t)(t - 1) * DV + tid] = u;
            }
        }
        if (nsteps == 0 && consumer_sync_or<kConsumers>(!ok)) abort = true;
        if (abort) break;

        if constexpr (COMMIT) {
            consumer_sync<kConsumers>();
            // C1: S_n = S^_0 e^{L_n} + sum_m u_m (k~_m e^{L_n - L_m})^T  (FP32, registers)
            const int nrec = pos + nsteps;
            float *gW_s = sc.gk, *cgW_s = sc.xk;
            for (int j = tid; j < DK; j += kConsumers) {
                const float Ln = GATE == 1 ? recL_s[(nrec - 1) * DK + j] : recL_s[nrec - 1];
                const float g = expf(Ln);
                gW_s[j] = g;
                cgW_s[j] = cs_s[j] * g;
            }
            if (GATE == 1) {
                for (int e = tid; e < nrec * DK; e += kConsumers) {
                    const int m = e / DK, j = e % DK;
                    recK_s[e] *= expf(recL_s[(nrec - 1) * DK + j] - recL_s[m * DK + j]);
                }
            } else {
                // one decay factor per record
                for (int e = tid; e < nrec * DK; e += kConsumers) {
                    const int m = e / DK;
                    recK_s[e] *= expf(recL_s[nrec - 1] - recL_s[m]);
                }
            }
            consumer_sync<kConsumers>();
            float Sreg[T::NR][4];
            {
                float cg[4];
                *reinterpret_cast<float4 *>(cg) = *reinterpret_cast<const float4 *>(cgW_s + c0);
#pragma unroll
                for (int n = 0; n < T::NR; ++n) {
                    const int row = T::row(warp, lane, n);
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(codes_s + row * DK + c0);
                    float f[4];
                    codes4_to_f32(w, f);
                    const float si = sig_s[row];
#pragma unroll
                    for (int e = 0; e < 4; ++e) Sreg[n][e] = (si * f[e]) * cg[e];
                }
                for (int c = 0; c < R; ++c) {
                    const int rc = compr_s[c];
#pragma unroll
                    for (int n = 0; n < T::NR; ++n)
                        if (T::row(warp, lane, n) == rc)
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                Sreg[n][e] = fmaf(compv_s[c * DK + c0 + e], gW_s[c0 + e], Sreg[n][e]);
                }
#pragma unroll 2
                for (int m = 0; m < nrec; ++m) {
                    float kh[4];
                    *reinterpret_cast<float4 *>(kh) =
                        *reinterpret_cast<const float4 *>(recK_s + m * DK + c0);
                    float u[T::NR];
                    if constexpr (T::RPI == 1 && T::NR % 4 == 0) {
                        // this lane's rows are consecutive: vector loads
#pragma unroll
                        for (int n = 0; n < T::NR; n += 4)
                            *reinterpret_cast<float4 *>(&u[n]) = *reinterpret_cast<const float4 *>(
                                recU_s + m * DV + T::row(warp, lane, n));
                    } else {
#pragma unroll
                        for (int n = 0; n < T::NR; ++n) u[n] = recU_s[m * DV + T::row(warp, lane, n)];
                    }
#pragma unroll
                    for (int n = 0; n < T::NR; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) Sreg[n][e] = fmaf(u[n], kh[e], Sreg[n][e]);
                }
            }
            SnapPtr out{a.codes + (size_t)bh * DV * DK, a.row_scale + (size_t)bh * DV,
                        a.col_smooth + (size_t)bh * DK,
                        a.comp_row ? a.comp_row + (size_t)bh * R : nullptr,
                        a.comp_val ? a.comp_val + (size_t)bh * R * DK : nullptr};
            quantize_tile<DK, DV, kConsumerWarps>(Sreg, R, a.smoothing != 0, sc.quant, out);
        }
        // release the stage to the producer
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

template <int DK, int DV, int GATE, bool BF16, bool COMMIT>
struct Launcher {
    static cudaError_t run(const DecodeArgs &a, cudaStream_t stream) {
        constexpr int E = BF16 ? 2 : 4;
        static std::atomic<uint64_t> configured{0};  // devices already set up
        static int sm_count[64];
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        auto kern = decode_kernel<DK, DV, GATE, BF16, COMMIT>;
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
        const StageLayout SL = stage_layout(DK, DV, GATE, a.R, a.W, E);
        const int fixed = header_bytes() + (int)sizeof(Scratch<DK, DV>);
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
};

template <int DK, int DV, int GATE, bool BF16>
cudaError_t launch_decode_c(const DecodeArgs &a, bool commit, cudaStream_t stream) {
    return commit ? Launcher<DK, DV, GATE, BF16, true>::run(a, stream)
                  : Launcher<DK, DV, GATE, BF16, false>::run(a, stream);
}

template <int DK, int DV>
cudaError_t launch_decode_d(const DecodeArgs &a, int gate, bool bf16, bool commit,
                            cudaStream_t stream) {
    if (gate == 1)
        return bf16 ? launch_decode_c<DK, DV, 1, true>(a, commit, stream)
                    : launch_decode_c<DK, DV, 1, false>(a, commit, stream);
    return bf16 ? launch_decode_c<DK, DV, 0, true>(a, commit, stream)
                : launch_decode_c<DK, DV, 0, false>(a, commit, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, int d_k, int d_v, int gate, bool bf16, bool commit,
                          cudaStream_t stream) {
    if (d_k == 128 && d_v == 128) return launch_decode_d<128, 128>(a, gate, bf16, commit, stream);
    if (d_k == 128 && d_v == 64) return launch_decode_d<128, 64>(a, gate, bf16, commit, stream);
    if (d_k == 64 && d_v == 128) return launch_decode_d<64, 128>(a, gate, bf16, commit, stream);
    if (d_k == 64 && d_v == 64) return launch_decode_d<64, 64>(a, gate, bf16, commit, stream);
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
