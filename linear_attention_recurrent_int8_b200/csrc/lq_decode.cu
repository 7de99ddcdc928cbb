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
// One CTA (8 warps) per (sequence, head).  Thread 0 stages the head's int8
// codes, scales, smoothing factors, compensators and buffered records into
// shared memory with bulk asynchronous copies (one mbarrier, bounded wait);
// the codes are dequantized in registers and multiplied against two vectors
// at once (FP32 FMA), and the two dot products of each row are reduced with a
// transposing warp reduction.  When the window fills (or for a standalone
// commit, launched with no tokens) the same CTA rebuilds the FP32 state in
// registers and re-quantizes it in place (lq_quant.cuh).
#include <atomic>

#include "lq_kernels.h"
#include "lq_quant.cuh"

namespace lq {

__device__ unsigned int g_dev_error = 0;

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }

// Byte offsets of the dynamic shared memory regions.
struct DecodeLayout {
    int bar, codes, sig, cs, compv, compr, recK, recU, recL, qk, xk, coef, y, misc, quant, total;
};

__host__ __device__ inline DecodeLayout decode_layout(int DK, int DV, int G, int R, int W,
                                                     int quant_bytes) {
    DecodeLayout L{};
    int o = 0;
    L.bar = o;   o += 16;
    L.codes = o; o += align16(DV * DK);
    L.sig = o;   o += align16(4 * DV);
    L.cs = o;    o += align16(4 * DK);
    L.compv = o; o += align16(4 * R * DK);
    L.compr = o; o += align16(4 * kMaxComp);
    L.recK = o;  o += align16(4 * W * DK);
    L.recU = o;  o += align16(4 * W * DV);
    L.recL = o;  o += align16(4 * W * G);
    L.qk = o;    o += align16(4 * 4 * DK);   // q, k, gk (e^L k), gq (e^L q)
    L.xk = o;    o += align16(4 * 3 * DK);   // xk = c gk, xq = c gq, k~
    L.coef = o;  o += align16(4 * 2 * (32 + kMaxComp + 1));
    L.y = o;     o += align16(4 * 2 * DV);
    L.misc = o;  o += 64;
    L.quant = o; o += align16(quant_bytes);
    L.total = o;
    return L;
}

template <int DK, int DV, int GATE, bool BF16, bool COMMIT>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeArgs a) {
    using T = Tile<DK, DV, kWarps>;
    constexpr int G = GATE == 1 ? DK : 1;
    extern __shared__ __align__(16) unsigned char smem[];
    const DecodeLayout L = decode_layout(DK, DV, G, a.R, a.W, sizeof(QuantSmem<DK, DV, kWarps>));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bar);
    int8_t *codes_s = reinterpret_cast<int8_t *>(smem + L.codes);
    float *sig_s = reinterpret_cast<float *>(smem + L.sig);
    float *cs_s = reinterpret_cast<float *>(smem + L.cs);
    float *compv_s = reinterpret_cast<float *>(smem + L.compv);
    int *compr_s = reinterpret_cast<int *>(smem + L.compr);
    float *recK_s = reinterpret_cast<float *>(smem + L.recK);
    float *recU_s = reinterpret_cast<float *>(smem + L.recU);
    float *recL_s = reinterpret_cast<float *>(smem + L.recL);
    float *q_s = reinterpret_cast<float *>(smem + L.qk);
    float *k_s = q_s + DK;
    float *gk_s = q_s + 2 * DK;
    float *gq_s = q_s + 3 * DK;
    float *xk_s = reinterpret_cast<float *>(smem + L.xk);
    float *xq_s = xk_s + DK;
    float *kt_s = xk_s + 2 * DK;
    float *coefA_s = reinterpret_cast<float *>(smem + L.coef);
    float *coefG_s = coefA_s + (32 + kMaxComp + 1);
    float *y_s = reinterpret_cast<float *>(smem + L.y);
    float *misc_s = reinterpret_cast<float *>(smem + L.misc);
    auto &qsm = *reinterpret_cast<QuantSmem<DK, DV, kWarps> *>(smem + L.quant);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H;
    const int R = a.R, W = a.W, pos = a.pos, nsteps = a.n_steps;

    const int8_t *codes_g = a.codes + (size_t)bh * DV * DK;
    const float *sig_g = a.row_scale + (size_t)bh * DV;
    const float *cs_g = a.col_smooth + (size_t)bh * DK;
    float *bufL = a.buf_gate + (size_t)bh * W * G;
    float *bufK = a.buf_k + (size_t)bh * W * DK;
    float *bufU = a.buf_u + (size_t)bh * W * DV;

    // ---- stage the head: bulk copies (thread 0) + small plain loads ----
    if (tid == 0) mbar_init(bar, 1);
    __syncthreads();
    if (tid == 0) {
        uint32_t bytes = DV * DK + 4 * DV + 4 * DK + 4 * R * DK + 4 * pos * (DK + DV) +
                         (GATE == 1 ? 4 * pos * DK : 0);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(codes_s, codes_g, DV * DK, bar);
        bulk_g2s(sig_s, sig_g, 4 * DV, bar);
        bulk_g2s(cs_s, cs_g, 4 * DK, bar);
        if (R > 0) bulk_g2s(compv_s, a.comp_val + (size_t)bh * R * DK, 4 * R * DK, bar);
        if (pos > 0) {
            bulk_g2s(recK_s, bufK, 4 * pos * DK, bar);
            bulk_g2s(recU_s, bufU, 4 * pos * DV, bar);
            if (GATE == 1) bulk_g2s(recL_s, bufL, 4 * pos * DK, bar);
        }
    }
    if (GATE == 0)
        for (int m = tid; m < pos; m += kThreads) recL_s[m] = bufL[m];
    if (tid < R) compr_s[tid] = a.comp_row[(size_t)bh * R + tid];
    const bool ok = mbar_wait_bounded(bar, 0);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) mbar_wait_bounded(bar, 0);
        return;
    }

    const int c0 = T::col0(lane);

    // ---- decode tokens at window positions pos+1 .. pos+nsteps ----
    for (int s = 0; s < nsteps; ++s) {
        const int t = pos + s + 1;
        const size_t tok = ((size_t)b * nsteps + s) * a.H + h;  // row of [B, n, H]
        const float beta = a.beta[tok];
        // D1: inputs, running log gate, k~
        if (tid < DK) {
            const float qj = load_io<BF16>(a.q, tok * DK + tid);
            const float kj = load_io<BF16>(a.k, tok * DK + tid);
            float Lt;
            if (GATE == 1) {
                const float prev = t > 1 ? recL_s[(t - 2) * DK + tid] : 0.0f;
                Lt = prev + logf(a.alpha[tok * DK + tid]);
                recL_s[(t - 1) * DK + tid] = Lt;
                bufL[(size_t)(t - 1) * DK + tid] = Lt;
            } else {
                const float prev = t > 1 ? recL_s[t - 2] : 0.0f;
                Lt = prev + logf(a.alpha[tok]);
                if (tid == 0) {
                    misc_s[0] = Lt;
                    recL_s[t - 1] = Lt;
                    bufL[t - 1] = Lt;
                }
            }
            const float g = expf(Lt);
            const float ktj = beta * kj;
            q_s[tid] = qj;
            k_s[tid] = kj;
            gk_s[tid] = g * kj;
            gq_s[tid] = g * qj;
            xk_s[tid] = cs_s[tid] * (g * kj);
            xq_s[tid] = cs_s[tid] * (g * qj);
            kt_s[tid] = ktj;
            recK_s[(t - 1) * DK + tid] = ktj;
            bufK[(size_t)(t - 1) * DK + tid] = ktj;
        }
        __syncthreads();

        // D3 coefficients: records 1..t-1, compensators, own token
        {
            const float Lt_s = GATE == 0 ? misc_s[0] : 0.0f;
            const int nrec = t - 1, nitems = nrec + R + 1;
            for (int it = warp; it < nitems; it += kWarps) {
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
                            da = fmaf(w, k_s[j], da);
                            dq = fmaf(w, q_s[j], dq);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < DK / 32; ++e) {
                            const int j = lane + 32 * e;
                            da = fmaf(km[j], k_s[j], da);
                            dq = fmaf(km[j], q_s[j], dq);
                        }
                    }
                    da = group_sum<32>(da);
                    dq = group_sum<32>(dq);
                    if (GATE == 0) {
                        const float dec = expf(Lt_s - recL_s[it]);
                        da *= dec;
                        dq *= dec;
                    }
                } else if (it < nrec + R) {
                    const float *cv = compv_s + (it - nrec) * DK;
#pragma unroll
                    for (int e = 0; e < DK / 32; ++e) {
                        const int j = lane + 32 * e;
                        da = fmaf(cv[j], gk_s[j], da);
                        dq = fmaf(cv[j], gq_s[j], dq);
                    }
                    da = group_sum<32>(da);
                    dq = group_sum<32>(dq);
                } else {
#pragma unroll
                    for (int e = 0; e < DK / 32; ++e) {
                        const int j = lane + 32 * e;
                        dq = fmaf(kt_s[j], q_s[j], dq);
                    }
                    dq = group_sum<32>(dq);
                }
                if (lane == 0) {
                    coefA_s[it] = da;
                    coefG_s[it] = dq;
                }
            }
        }

        // D2: y_k = Q (c e^L k), y_q = Q (c e^L q), two vectors per pass
        {
            float xk[4], xq[4];
            *reinterpret_cast<float4 *>(xk) = *reinterpret_cast<const float4 *>(xk_s + c0);
            *reinterpret_cast<float4 *>(xq) = *reinterpret_cast<const float4 *>(xq_s + c0);
            float acc[2 * T::NR];
#pragma unroll
            for (int n = 0; n < T::NR; ++n) {
                const int row = T::row(warp, lane, n);
                const uint32_t w = *reinterpret_cast<const uint32_t *>(codes_s + row * DK + c0);
                float f[4];
                codes4_to_f32(w, f);
                float ak = f[0] * xk[0], aq = f[0] * xq[0];
#pragma unroll
                for (int e = 1; e < 4; ++e) {
                    ak = fmaf(f[e], xk[e], ak);
                    aq = fmaf(f[e], xq[e], aq);
                }
                acc[n] = ak;
                acc[T::NR + n] = aq;
            }
            transposed_sum<2 * T::NR, T::LPR>(acc, lane);
            const int idx = transposed_index<2 * T::NR, T::LPR>(lane);
            const int vec = idx / T::NR, n = idx % T::NR;
            const int row = T::row(warp, lane, n);
            y_s[vec * DV + row] = acc[0] * sig_s[row];
        }
        __syncthreads();

        // D3-D6 per row: correction, u_t, o_t, record
        if (tid < DV) {
            const int i = tid;
            const int nrec = t - 1;
            float hb = y_s[i], p = y_s[DV + i];
            for (int c = 0; c < R; ++c)
                if (compr_s[c] == i) {
                    hb += coefA_s[nrec + c];
                    p += coefG_s[nrec + c];
                }
            for (int m = 0; m < nrec; ++m) {
                const float um = recU_s[m * DV + i];
                hb = fmaf(coefA_s[m], um, hb);
                p = fmaf(coefG_s[m], um, p);
            }
            const float u = load_io<BF16>(a.v, tok * DV + i) - hb;
            const float o = fmaf(coefG_s[nrec + R], u, p);
            store_io<BF16>(a.o, tok * DV + i, o);
            recU_s[(t - 1) * DV + i] = u;
            bufU[(size_t)(t - 1) * DV + i] = u;
        }
        __syncthreads();
    }

    if constexpr (COMMIT) {
        // C1: S_n = S^_0 e^{L_n} + sum_m u_m (k~_m e^{L_n - L_m})^T  (FP32, registers)
        const int nrec = pos + nsteps;
        float *gW_s = gk_s, *cgW_s = xk_s;
        for (int j = tid; j < DK; j += kThreads) {
            const float Ln = GATE == 1 ? recL_s[(nrec - 1) * DK + j] : recL_s[nrec - 1];
            const float g = expf(Ln);
            gW_s[j] = g;
            cgW_s[j] = cs_s[j] * g;
        }
        for (int e = tid; e < nrec * DK; e += kThreads) {
            const int m = e / DK, j = e % DK;
            const float Ln = GATE == 1 ? recL_s[(nrec - 1) * DK + j] : recL_s[nrec - 1];
            const float Lm = GATE == 1 ? recL_s[m * DK + j] : recL_s[m];
            recK_s[e] *= expf(Ln - Lm);
        }
        __syncthreads();
        float S[T::NR][4];
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
                for (int e = 0; e < 4; ++e) S[n][e] = (si * f[e]) * cg[e];
            }
            for (int c = 0; c < R; ++c) {
                const int rc = compr_s[c];
#pragma unroll
                for (int n = 0; n < T::NR; ++n)
                    if (T::row(warp, lane, n) == rc)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            S[n][e] = fmaf(compv_s[c * DK + c0 + e], gW_s[c0 + e], S[n][e]);
            }
            for (int m = 0; m < nrec; ++m) {
                float kh[4];
                *reinterpret_cast<float4 *>(kh) =
                    *reinterpret_cast<const float4 *>(recK_s + m * DK + c0);
#pragma unroll
                for (int n = 0; n < T::NR; ++n) {
                    const float u = recU_s[m * DV + T::row(warp, lane, n)];
#pragma unroll
                    for (int e = 0; e < 4; ++e) S[n][e] = fmaf(u, kh[e], S[n][e]);
                }
            }
        }
        // The old snapshot in shared memory has been read by every thread.
        __syncthreads();
        SnapPtr out{a.codes + (size_t)bh * DV * DK, a.row_scale + (size_t)bh * DV,
                    a.col_smooth + (size_t)bh * DK,
                    a.comp_row ? a.comp_row + (size_t)bh * R : nullptr,
                    a.comp_val ? a.comp_val + (size_t)bh * R * DK : nullptr};
        quantize_tile<DK, DV, kWarps>(S, R, a.smoothing != 0, qsm, out);
    }
}

// Opts a kernel into its largest possible dynamic shared memory (W = 32,
// r = 16) once per device; launches then pass their actual size.  `done`
// is the caller's per-kernel record of the devices already set up.
template <typename K>
cudaError_t opt_in_smem(K kern, int max_bytes, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

template <int DK, int DV, int GATE, bool BF16, bool COMMIT>
cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t stream) {
    constexpr int G = GATE == 1 ? DK : 1;
    constexpr int QB = sizeof(QuantSmem<DK, DV, kWarps>);
    const DecodeLayout L = decode_layout(DK, DV, G, a.R, a.W, QB);
    auto kern = decode_kernel<DK, DV, GATE, BF16, COMMIT>;
    static std::atomic<uint64_t> done{0};  // one per kernel instantiation
    cudaError_t e = opt_in_smem(kern, decode_layout(DK, DV, G, kMaxComp, 32, QB).total, done);
    if (e != cudaSuccess) return e;
    kern<<<a.B * a.H, kThreads, L.total, stream>>>(a);
    return cudaGetLastError();
}

template <int DK, int DV, int GATE, bool BF16>
cudaError_t launch_decode_c(const DecodeArgs &a, bool commit, cudaStream_t stream) {
    return commit ? launch_decode_t<DK, DV, GATE, BF16, true>(a, stream)
                  : launch_decode_t<DK, DV, GATE, BF16, false>(a, stream);
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

int decode_smem_bytes(int d_k, int d_v, int gate, int R, int W) {
    const int G = gate == 1 ? d_k : 1;
    int q = 0;
    if (d_k == 128 && d_v == 128) q = sizeof(QuantSmem<128, 128, kWarps>);
    if (d_k == 128 && d_v == 64) q = sizeof(QuantSmem<128, 64, kWarps>);
    if (d_k == 64 && d_v == 128) q = sizeof(QuantSmem<64, 128, kWarps>);
    if (d_k == 64 && d_v == 64) q = sizeof(QuantSmem<64, 64, kWarps>);
    return decode_layout(d_k, d_v, G, R, W, q).total;
}

}  // namespace lq
