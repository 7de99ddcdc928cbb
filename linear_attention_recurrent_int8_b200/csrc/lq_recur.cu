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
#include <atomic>

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

// Long runs (prefill): the same ownership (a lane holds 4 key channels of
// each of its warp's rows, so each token vector is read once per warp with
// one load per lane), 8 rows per warp, and no shared-memory round trip
// inside the token loop: after the transposing reduction the lane that holds
// S_{t-1} b_t of a row forms u_t, passes it by shuffle to the lane that holds
// S_{t-1} (alpha q_t) (which writes o_t), and every lane fetches the rows'
// u_t by shuffle for its update.  The tokens' raw inputs arrive in chunks of
// 16 by 16-byte cp.async copies into a second buffer while the current
// chunk is computed, so no load latency sits on the token loop.
template <int DK, int DV, int GATE, bool BF16, int NWARPS, int RW>
struct RowsSmem {
    static constexpr int E = BF16 ? 2 : 4, G = GATE == 1 ? DK : 1, RPC = NWARPS * RW;
    alignas(16) unsigned char k[2][kChunk][DK * E];
    alignas(16) unsigned char q[2][kChunk][DK * E];
    alignas(16) unsigned char v[2][kChunk][RPC * E];
    alignas(16) float al[2][kChunk][G];
    alignas(16) float beta[2][kChunk];
    float kq[2][kChunk];
};

template <int DK, int DV, int GATE, bool BF16, int NWARPS, int RW>
__global__ void __launch_bounds__(NWARPS * 32) recur_rows_kernel(const RecurArgs a) {
    using Sm = RowsSmem<DK, DV, GATE, BF16, NWARPS, RW>;
    constexpr int E = Sm::E;
    constexpr int LPR = DK / 4, RPI = 32 / LPR, NR = RW / RPI, RPC = NWARPS * RW;
    constexpr int NT = NWARPS * 32;
    static_assert(DV % RPC == 0, "bad row split");
    extern __shared__ __align__(16) unsigned char rows_smem[];
    Sm &sm = *reinterpret_cast<Sm *>(rows_smem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int cph = DV / RPC;
    const int bh = blockIdx.x / cph;
    const int rbase = (blockIdx.x % cph) * RPC;
    const int b = bh / a.H, h = bh % a.H;
    const int c0 = 4 * (lane % LPR);
    const int rs = lane / LPR;
    const int idx = transposed_index<2 * NR, LPR>(lane);  // the value this lane holds after the reduction
    const int gbase = lane & ~(LPR - 1);

    auto tok_of = [&](int t) { return ((size_t)b * a.T_total + a.t0 + t) * a.H + h; };
    // raw copies of tokens [t, t + n) into buffer p
    auto stage = [&](int p, int t, int n) {
        const unsigned char *kg = static_cast<const unsigned char *>(a.k);
        const unsigned char *qg = static_cast<const unsigned char *>(a.q);
        const unsigned char *vg = static_cast<const unsigned char *>(a.v);
        constexpr int KC = DK * E / 16, VC = RPC * E / 16;
        for (int i = tid; i < n * KC; i += NT) {
            const int tt = i / KC, c = i % KC;
            const size_t tok = tok_of(t + tt);
            cp_async16(&sm.k[p][tt][16 * c], kg + tok * DK * E + 16 * c);
            cp_async16(&sm.q[p][tt][16 * c], qg + tok * DK * E + 16 * c);
        }
        for (int i = tid; i < n * VC; i += NT) {
            const int tt = i / VC, c = i % VC;
            cp_async16(&sm.v[p][tt][16 * c], vg + (tok_of(t + tt) * DV + rbase) * E + 16 * c);
        }
        if (GATE == 1) {
            for (int i = tid; i < n * (DK / 4); i += NT) {
                const int tt = i / (DK / 4), c = i % (DK / 4);
                cp_async16(&sm.al[p][tt][4 * c], a.alpha + tok_of(t + tt) * DK + 4 * c);
            }
        } else {
            for (int tt = tid; tt < n; tt += NT) cp_async4(&sm.al[p][tt][0], a.alpha + tok_of(t + tt));
        }
        for (int tt = tid; tt < n; tt += NT) cp_async4(&sm.beta[p][tt], a.beta + tok_of(t + tt));
        cp_async_commit();
    };
    auto load4 = [&](const unsigned char *row, int j, float (&x)[4]) {
        if constexpr (BF16) {
            const uint2 w = *reinterpret_cast<const uint2 *>(row + 2 * j);
            x[0] = __uint_as_float(w.x << 16);
            x[1] = __uint_as_float(w.x & 0xFFFF0000u);
            x[2] = __uint_as_float(w.y << 16);
            x[3] = __uint_as_float(w.y & 0xFFFF0000u);
        } else {
            *reinterpret_cast<float4 *>(x) = *reinterpret_cast<const float4 *>(row + 4 * j);
        }
    };
    auto load1 = [&](const unsigned char *row, int j) -> float {
        if constexpr (BF16)
            return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(row)[j]);
        else
            return reinterpret_cast<const float *>(row)[j];
    };
    // k~ . q of the staged tokens: one warp per token
    auto kq_of = [&](int p, int n) {
        for (int tt = warp; tt < n; tt += NWARPS) {
            float d = 0.0f;
#pragma unroll
            for (int e = 0; e < DK / 32; ++e)
                d = fmaf(load1(sm.k[p][tt], lane + 32 * e), load1(sm.q[p][tt], lane + 32 * e), d);
            d = group_sum<32>(d);
            if (lane == 0) sm.kq[p][tt] = sm.beta[p][tt] * d;
        }
    };

    float S[NR][4];
    float *Sg = a.S + ((size_t)bh * DV + rbase) * DK;
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const float4 x = *reinterpret_cast<const float4 *>(Sg + (size_t)(warp * RW + n * RPI + rs) * DK + c0);
        S[n][0] = x.x;
        S[n][1] = x.y;
        S[n][2] = x.z;
        S[n][3] = x.w;
    }

    const int nt = a.nt;
    if (nt > 0) {
        stage(0, 0, min(kChunk, nt));
        cp_async_wait_all();
        __syncthreads();
        kq_of(0, min(kChunk, nt));
        __syncthreads();
    }
    for (int tc0 = 0, p = 0; tc0 < nt; tc0 += kChunk, p ^= 1) {
        const int nc = min(kChunk, nt - tc0);
        const int nn = min(kChunk, nt - tc0 - nc);
        if (nn > 0) stage(p ^ 1, tc0 + nc, nn);
        for (int tt = 0; tt < nc; ++tt) {
            float k4[4], q4[4], a4[4], b4[4];
            load4(sm.k[p][tt], c0, k4);
            load4(sm.q[p][tt], c0, q4);
            if (GATE == 1) {
                *reinterpret_cast<float4 *>(a4) = *reinterpret_cast<const float4 *>(&sm.al[p][tt][c0]);
            } else {
                a4[0] = a4[1] = a4[2] = a4[3] = sm.al[p][tt][0];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                b4[e] = a.delta ? a4[e] * k4[e] : 0.0f;
                q4[e] *= a4[e];
            }
            float acc[2 * NR];
            const float2 b01 = make_float2(b4[0], b4[1]), b23 = make_float2(b4[2], b4[3]);
            const float2 q01 = make_float2(q4[0], q4[1]), q23 = make_float2(q4[2], q4[3]);
#pragma unroll
            for (int n = 0; n < NR; ++n) {
                const float2 s01 = make_float2(S[n][0], S[n][1]), s23 = make_float2(S[n][2], S[n][3]);
                const float2 hb = __ffma2_rn(s23, b23, __fmul2_rn(s01, b01));
                const float2 pp = __ffma2_rn(s23, q23, __fmul2_rn(s01, q01));
                acc[n] = hb.x + hb.y;
                acc[NR + n] = pp.x + pp.y;
            }
            transposed_sum<2 * NR, LPR>(acc, lane);
            const int rloc = (idx % NR) * RPI + rs;  // warp-local row of this lane's value
            float u = 0.0f;
            if (idx < NR) u = load1(sm.v[p][tt], warp * RW + rloc) - acc[0];
            const float u_row = __shfl_sync(0xffffffffu, u, gbase + transposed_owner<2 * NR, LPR>(idx % NR));
            if (idx >= NR && lane == gbase + transposed_owner<2 * NR, LPR>(idx))
                store_io<BF16>(a.o, tok_of(tc0 + tt) * DV + rbase + warp * RW + rloc,
                               fmaf(sm.kq[p][tt], u_row, acc[0]));
            const float beta = sm.beta[p][tt];
            const float2 kt01 = make_float2(beta * k4[0], beta * k4[1]);
            const float2 kt23 = make_float2(beta * k4[2], beta * k4[3]);
            const float2 a01 = make_float2(a4[0], a4[1]), a23 = make_float2(a4[2], a4[3]);
#pragma unroll
            for (int n = 0; n < NR; ++n) {
                const float un = __shfl_sync(0xffffffffu, u, gbase + transposed_owner<2 * NR, LPR>(n));
                const float2 u2 = make_float2(un, un);
                const float2 s01 = __ffma2_rn(make_float2(S[n][0], S[n][1]), a01, __fmul2_rn(u2, kt01));
                const float2 s23 = __ffma2_rn(make_float2(S[n][2], S[n][3]), a23, __fmul2_rn(u2, kt23));
                S[n][0] = s01.x;
                S[n][1] = s01.y;
                S[n][2] = s23.x;
                S[n][3] = s23.y;
            }
        }
        if (nn > 0) {
            cp_async_wait_all();
            __syncthreads();  // the next chunk has arrived; this chunk's buffer is free
            kq_of(p ^ 1, nn);
            __syncthreads();
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
        // 4 warps x 8 rows: DV/32 CTAs per head (4 rows per warp measured slower)
        constexpr int NW = 4, RW = 8;
        constexpr int smem = (int)sizeof(RowsSmem<DK, DV, GATE, BF16, NW, RW>);
        auto kern = recur_rows_kernel<DK, DV, GATE, BF16, NW, RW>;
        static std::atomic<uint64_t> configured{0};  // devices already set up
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const uint64_t bit = 1ull << (dev & 63);
        if (!(configured.load(std::memory_order_acquire) & bit)) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            configured.fetch_or(bit, std::memory_order_acq_rel);
        }
        kern<<<a.B * a.H * (DV / (NW * RW)), NW * 32, smem, stream>>>(a);
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
