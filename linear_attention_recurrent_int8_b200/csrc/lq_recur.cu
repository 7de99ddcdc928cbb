// lq_recur.cu -- the recurrence on an FP32 state, token by token:
//   S_t = S_{t-1} D_t + (v_t - S_{t-1} b_t) k~_t^T,   o_t = S_t q_t
// (equation 1 of "LeapQuant: Efficient Linear Attention with Accurate
// Recurrent State Quantization", Appendix Table 4; Gated DeltaNet and the
// diagonal Kimi-Delta-Attention gate).
//
// Two uses:
//  * prefill: a long run of tokens from a caller FP32 state (the state is
//    carried in FP32; snapshots are quantized copies taken between launches);
//  * the FP32 per-step comparator of the paper's Table 2, where the whole
//    FP32 state is read and written every step.
//
// Rows of S evolve independently given (k, q, alpha, beta), so a CTA owns a
// slice of rows held in registers (each lane 4 key channels of a few rows).
// Per token both dot products S_{t-1} (alpha*k) and S_{t-1} (alpha*q) are
// formed in one pass and reduced with a transposing warp reduction; then
// u = v - S b, o = S_{t-1}(alpha*q) + u (k~ . q), S = S Diag(alpha) + u k~^T.
// Inputs are staged through shared memory in chunks of tokens.
#include "lq_common.cuh"
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kChunk = 16;

template <int DK, int DV, int GATE, bool BF16, int NWARPS, int RW>
__global__ void __launch_bounds__(NWARPS * 32) recur_kernel(const RecurArgs a) {
    constexpr int LPR = DK / 4, RPI = 32 / LPR, NR = RW / RPI, RPC = NWARPS * RW;
    constexpr int NT = NWARPS * 32;
    constexpr int G = GATE == 1 ? DK : 1;
    static_assert(RW % RPI == 0 && RW <= 32 && DV % RPC == 0, "bad row split");
    __shared__ __align__(16) float k_s[kChunk][DK];
    __shared__ __align__(16) float q_s[kChunk][DK];
    __shared__ __align__(16) float a_s[kChunk][G];
    __shared__ float v_s[kChunk][RPC];
    __shared__ float beta_s[kChunk], kq_s[kChunk];
    __shared__ float y_s[NWARPS][2][RW];
    __shared__ float u_s[NWARPS][RW];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int cph = DV / RPC;
    const int bh = blockIdx.x / cph;
    const int rbase = (blockIdx.x % cph) * RPC;
    const int b = bh / a.H, h = bh % a.H;
    const int c0 = 4 * (lane % LPR);
    const int rs = lane / LPR;

    float S[NR][4];
    float *Sg = a.S + ((size_t)bh * DV + rbase) * DK;
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const float4 x =
            *reinterpret_cast<const float4 *>(Sg + (size_t)(warp * RW + n * RPI + rs) * DK + c0);
        S[n][0] = x.x;
        S[n][1] = x.y;
        S[n][2] = x.z;
        S[n][3] = x.w;
    }

    for (int tc0 = 0; tc0 < a.nt; tc0 += kChunk) {
        const int nc = min(kChunk, a.nt - tc0);
        __syncthreads();
        for (int i = tid; i < nc * DK; i += NT) {
            const int tt = i / DK, j = i % DK;
            const size_t tok = ((size_t)b * a.T_total + a.t0 + tc0 + tt) * a.H + h;
            k_s[tt][j] = load_io<BF16>(a.k, tok * DK + j);
            q_s[tt][j] = load_io<BF16>(a.q, tok * DK + j);
            if (GATE == 1) a_s[tt][j] = a.alpha[tok * DK + j];
        }
        for (int i = tid; i < nc * RPC; i += NT) {
            const int tt = i / RPC, r = i % RPC;
            const size_t tok = ((size_t)b * a.T_total + a.t0 + tc0 + tt) * a.H + h;
            v_s[tt][r] = load_io<BF16>(a.v, tok * DV + rbase + r);
        }
        for (int tt = tid; tt < nc; tt += NT) {
            const size_t tok = ((size_t)b * a.T_total + a.t0 + tc0 + tt) * a.H + h;
            beta_s[tt] = a.beta[tok];
            if (GATE == 0) a_s[tt][0] = a.alpha[tok];
        }
        __syncthreads();
        // k~ . q per token
        for (int tt = warp; tt < nc; tt += NWARPS) {
            float d = 0.0f;
#pragma unroll
            for (int e = 0; e < DK / 32; ++e) d = fmaf(k_s[tt][lane + 32 * e], q_s[tt][lane + 32 * e], d);
            d = group_sum<32>(d);
            if (lane == 0) kq_s[tt] = beta_s[tt] * d;
        }
        __syncthreads();

        for (int tt = 0; tt < nc; ++tt) {
            float k4[4], q4[4], a4[4];
            *reinterpret_cast<float4 *>(k4) = *reinterpret_cast<const float4 *>(&k_s[tt][c0]);
            *reinterpret_cast<float4 *>(q4) = *reinterpret_cast<const float4 *>(&q_s[tt][c0]);
            if (GATE == 1) {
                *reinterpret_cast<float4 *>(a4) = *reinterpret_cast<const float4 *>(&a_s[tt][c0]);
            } else {
                a4[0] = a4[1] = a4[2] = a4[3] = a_s[tt][0];
            }
            float b4[4];  // b_t = alpha (.) k_t, or 0 for the b = 0 rows
#pragma unroll
            for (int e = 0; e < 4; ++e) b4[e] = a.delta ? a4[e] * k4[e] : 0.0f;
            float acc[2 * NR];
#pragma unroll
            for (int n = 0; n < NR; ++n) {
                float hb = S[n][0] * b4[0], pp = S[n][0] * (a4[0] * q4[0]);
#pragma unroll
                for (int e = 1; e < 4; ++e) {
                    hb = fmaf(S[n][e], b4[e], hb);
                    pp = fmaf(S[n][e], a4[e] * q4[e], pp);
                }
                acc[n] = hb;
                acc[NR + n] = pp;
            }
            transposed_sum<2 * NR, LPR>(acc, lane);
            {
                const int idx = transposed_index<2 * NR, LPR>(lane);
                y_s[warp][idx / NR][(idx % NR) * RPI + rs] = acc[0];
            }
            __syncwarp();
            if (lane < RW) {
                const float u = v_s[tt][warp * RW + lane] - y_s[warp][0][lane];
                const float o = fmaf(kq_s[tt], u, y_s[warp][1][lane]);
                const size_t tok = ((size_t)b * a.T_total + a.t0 + tc0 + tt) * a.H + h;
                store_io<BF16>(a.o, tok * DV + rbase + warp * RW + lane, o);
                u_s[warp][lane] = u;
            }
            __syncwarp();
            const float beta = beta_s[tt];
#pragma unroll
            for (int n = 0; n < NR; ++n) {
                const float u = u_s[warp][n * RPI + rs];
#pragma unroll
                for (int e = 0; e < 4; ++e) S[n][e] = fmaf(S[n][e], a4[e], u * (beta * k4[e]));
            }
            __syncwarp();
        }
    }

#pragma unroll
    for (int n = 0; n < NR; ++n)
        *reinterpret_cast<float4 *>(Sg + (size_t)(warp * RW + n * RPI + rs) * DK + c0) =
            make_float4(S[n][0], S[n][1], S[n][2], S[n][3]);
}

template <int DK, int DV, int GATE, bool BF16>
cudaError_t launch_r(const RecurArgs &a, bool long_run, cudaStream_t stream) {
    if (long_run) {
        // 4 warps x 4 rows: DV/16 CTAs per head
        constexpr int NW = 4, RW = 4;
        recur_kernel<DK, DV, GATE, BF16, NW, RW>
            <<<a.B * a.H * (DV / (NW * RW)), NW * 32, 0, stream>>>(a);
    } else {
        // one CTA of 8 warps per head
        constexpr int NW = 8, RW = DV / 8;
        recur_kernel<DK, DV, GATE, BF16, NW, RW><<<a.B * a.H, NW * 32, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_r_d(const RecurArgs &a, int gate, bool bf16, bool long_run,
                       cudaStream_t stream) {
    if (gate == 1)
        return bf16 ? launch_r<DK, DV, 1, true>(a, long_run, stream)
                    : launch_r<DK, DV, 1, false>(a, long_run, stream);
    return bf16 ? launch_r<DK, DV, 0, true>(a, long_run, stream)
                : launch_r<DK, DV, 0, false>(a, long_run, stream);
}

}  // namespace

cudaError_t launch_recurrence(const RecurArgs &a, int d_k, int d_v, int gate, bool bf16,
                              bool long_run, cudaStream_t stream) {
    if (d_k == 128 && d_v == 128) return launch_r_d<128, 128>(a, gate, bf16, long_run, stream);
    if (d_k == 128 && d_v == 64) return launch_r_d<128, 64>(a, gate, bf16, long_run, stream);
    if (d_k == 64 && d_v == 128) return launch_r_d<64, 128>(a, gate, bf16, long_run, stream);
    if (d_k == 64 && d_v == 64) return launch_r_d<64, 64>(a, gate, bf16, long_run, stream);
    return cudaErrorInvalidValue;
}

}  // namespace lq
