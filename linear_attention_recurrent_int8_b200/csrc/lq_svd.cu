// lq_svd.cu -- the rank-r SVD compensator rule (lq_comp_rule LQ_COMP_SVD).
//
// "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
// Quantization", Abstract and Figure 4: the state's largest outliers are kept
// in high precision as Compensator Tokens, which share the update path of the
// real tokens, and the rest is smoothed and quantized.  The pages do not fix
// how the outliers are chosen.  This file implements the library's second
// rule: the r largest singular triplets of the FP32 state S (d_v x d_k),
// kept as the rank-one pseudo-records u_c k~_c^T with u_c = s_c U_c and
// k~_c = V_c (the largest-magnitude entry of k~_c positive), so that the
// residual S - sum_c u_c k~_c^T is the best rank-r-deflated state; the residual
// then goes through residual smoothing and per-row codes (C3-C4 of
// lq_quant.cuh, with no row compensators).
//
// One CTA of 512 threads per head, everything in shared memory:
//  1. S: the FP32 state (state initialisation, prefill snapshots), or its
//     rebuild at a window commit, S_n = S^_0 D_{1..n} + sum_m u_m K^_m^T
//     over the n buffered records and the old compensators;
//  2. G = S^T S (d_k x d_k, FP32, register-blocked);
//  3. subspace iteration on G with P = r + 8 basis vectors (rounded up to 4,
//     at most d_k): deterministic start vectors, or at a commit the old
//     compensators' k~_c in the first r columns; 16 steps V <- orth(G V),
//     each orthonormalised by classical Gram-Schmidt applied twice (FP32,
//     four CTA barriers per column);
//  4. Rayleigh-Ritz: H = V^T G V (FP64), its eigenvectors by a cyclic Jacobi
//     method with the round-robin pair ordering (P/2 rotations per round,
//     FP64; sweeps until the off-diagonal part is at round-off, at most 8),
//     the r largest; k~_c = V z_c, u_c = S k~_c;
//  5. the residual S - sum_c u_c k~_c^T into the register tile and C3-C4.
// The convergence rate of step 3 is (s_{P+1} / s_r)^2 per step.  A commit's
// rebuilt state is dominated by the W buffered rank-one records, so P > W
// converges in a few steps there; for a dense random state with nearly equal
// singular values around s_r the individual vectors of that cluster are not
// determined (by any method), only the singular values and a valid
// decomposition are.
#include "lq_kernels.h"
#include "lq_quant.cuh"

namespace lq {
namespace {

constexpr int kSWarps = 16, kSThreads = kSWarps * 32;
constexpr int kMaxP = 24;        // basis vectors
constexpr int kSteps = 16;       // subspace-iteration steps
constexpr int kSweeps = 8;       // Jacobi sweeps of the Rayleigh-Ritz eigenproblem
constexpr int kMaxRec = 32;      // buffered records (W <= 32)

__host__ __device__ constexpr int max_i(int a, int b) { return a > b ? a : b; }

template <int DK, int DV>
struct SvdSmem {
    static constexpr int SP = DK + 4;  // row pitch of S and G (floats)
    // G, and before it the rebuild's operands: K^ [n + r][DK] then U [n + r][DV]
    static constexpr int GF = max_i(DK * SP, (kMaxRec + kMaxComp) * (DK + DV));
    alignas(16) float S[DV * SP];
    alignas(16) float G[GF];
    alignas(16) float V[DK * kMaxP];   // basis, element (j, c) at j * kMaxP + c
    alignas(16) float X[DK * kMaxP];   // G V
    double H[kMaxP * kMaxP];           // Rayleigh quotient, rotated in place
    double Z[kMaxP * kMaxP];           // its eigenvectors (columns)
    double rc[kMaxP / 2], rs[kMaxP / 2];
    int jacobi_done;                   // the off-diagonal part has vanished
    float dot[kMaxP];
    alignas(16) float uc[kMaxComp * DV];
    alignas(16) float vc[kMaxComp * DK];
    int order[kMaxP];
    QuantSmem<DK, DV, kSWarps> q;
};

template <int DK, int DV>
constexpr size_t svd_smem_bytes() {
    return sizeof(SvdSmem<DK, DV>);
}

__device__ __forceinline__ void cta_sync() { __syncthreads(); }

// A deterministic start vector entry in {-1, +1} / sqrt(d_k) (an integer hash
// of the channel and the column; no random state).
__device__ __forceinline__ float start_entry(int j, int c, int DK) {
    uint32_t h = (uint32_t)j * 0x9E3779B1u ^ ((uint32_t)c + 1u) * 0x85EBCA77u;
    h ^= h >> 15;
    h *= 0xC2B2AE3Du;
    h ^= h >> 13;
    return (h & 1u ? 1.0f : -1.0f) * rsqrtf((float)DK);
}

// Classical Gram-Schmidt applied twice to the columns of X (DK x P, pitch
// kMaxP), written to V: column c loses its components along V's columns
// 0..c-1 (twice), then is normalised.  Four CTA barriers per column: warp 0
// normalises column c-1 (and takes its dot product with column c) while the
// other warps form column c's first projections.  A column that vanishes
// exactly becomes 0.
template <int DK>
__device__ void orthonormalise(float *V, float *X, float *dot, int P) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int RPL = DK / 32;  // rows per lane in a one-warp column pass
    // warp 0: V[:, c] = X[:, c] / |X[:, c]|, then dot[c] = X[:, c + 1] . V[:, c]
    auto finalise = [&](int c, bool with_next) {
        float x[RPL], n2 = 0.0f;
#pragma unroll
        for (int t = 0; t < RPL; ++t) {
            x[t] = X[(lane + 32 * t) * kMaxP + c];
            n2 = fmaf(x[t], x[t], n2);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
        const float inv = n2 > 1e-30f ? rsqrtf(n2) : 0.0f;
        float d = 0.0f;
#pragma unroll
        for (int t = 0; t < RPL; ++t) {
            const int j = lane + 32 * t;
            const float v = x[t] * inv;
            V[j * kMaxP + c] = v;
            if (with_next) d = fmaf(v, X[j * kMaxP + c + 1], d);
        }
        if (with_next) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (lane == 0) dot[c] = d;
        }
    };
    // dot[k] = X[:, c] . V[:, k] for k in [0, kend), warps from `first` on
    auto dots = [&](int c, int kend, int first) {
        for (int k = warp - first; k < kend; k += kSWarps - first) {
            if (k < 0) continue;
            float d = 0.0f;
            for (int j = lane; j < DK; j += 32) d = fmaf(V[j * kMaxP + k], X[j * kMaxP + c], d);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (lane == 0) dot[k] = d;
        }
    };
    auto update = [&](int c) {
        for (int j = tid; j < DK; j += kSThreads) {
            float x = X[j * kMaxP + c];
            for (int k = 0; k < c; ++k) x = fmaf(-dot[k], V[j * kMaxP + k], x);
            X[j * kMaxP + c] = x;
        }
    };
    for (int c = 0; c < P; ++c) {
        // first pass: column c-1 is finalised by warp 0, which also takes
        // the projection on it; the other warps take columns 0..c-2
        if (c > 0) {
            if (warp == 0) finalise(c - 1, true);
            else dots(c, c - 1, 1);
            cta_sync();
            update(c);
            cta_sync();
            // second pass
            dots(c, c, 0);
            cta_sync();
            update(c);
            cta_sync();
        }
    }
    if (warp == 0) finalise(P - 1, false);
    cta_sync();
}

// Arguments: FP32 states (S != nullptr), or a rebuild from the snapshot and
// the d.pos buffered records (a window commit; with d.seq_pos set, only the
// heads of sequences whose position equals d.commit_match).
struct SvdArgs {
    const float *S;
    DecodeArgs d;
};

template <int DK, int DV, int GATE, int FMT>
__global__ void __launch_bounds__(kSThreads, 1) svd_kernel(const SvdArgs A) {
    using T = Tile<DK, DV, kSWarps>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<SvdSmem<DK, DV> *>(smem_raw);
    constexpr int SP = SvdSmem<DK, DV>::SP;
    constexpr bool PACK4 = FMT == kCodesI4, BF16S = FMT == kCodesBF16;
    constexpr int CRB = code_row_bytes(FMT, DK);
    const DecodeArgs &a = A.d;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int R = a.R, W = a.W;
    if (A.S == nullptr && a.seq_pos && a.seq_pos[bh / a.H] != a.commit_match) return;
    const bool rebuild = A.S == nullptr;
    const int n = rebuild ? a.pos : 0;  // buffered records
    const int P = min(DK, ((R + 8) + 3) & ~3);
    const int8_t *codes = a.codes + (size_t)bh * DV * CRB;

    // ---------------------------------------------------------------- 1. S
    if (!rebuild) {
        for (int idx = tid; idx < DV * DK / 4; idx += kSThreads) {
            const int i = idx / (DK / 4), j = 4 * (idx % (DK / 4));
            *reinterpret_cast<float4 *>(&sm.S[i * SP + j]) =
                *reinterpret_cast<const float4 *>(A.S + ((size_t)bh * DV + i) * DK + j);
        }
        for (int idx = tid; idx < DK * P; idx += kSThreads) {
            const int j = idx / P, c = idx % P;
            sm.X[j * kMaxP + c] = start_entry(j, c, DK);
        }
    } else {
        // operands K^ (decayed records, then compensators times e^{L_n}) and U
        float *KH = sm.G;
        float *UU = sm.G + (n + R) * DK;
        const size_t gb = (size_t)bh * W * (GATE == 1 ? DK : 1);
        auto Lg = [&](int m, int j) { return a.buf_gate[gb + (size_t)m * (GATE == 1 ? DK : 1) + (GATE == 1 ? j : 0)]; };
        for (int idx = tid; idx < (n + R) * DK; idx += kSThreads) {
            const int m = idx / DK, j = idx % DK;
            const float Ln = Lg(n - 1, j);
            float x;
            if (m < n) x = a.buf_k[((size_t)bh * W + m) * DK + j] * expf(Ln - Lg(m, j));
            else x = a.comp_val[((size_t)bh * R + (m - n)) * DK + j] * expf(Ln);
            KH[idx] = x;
        }
        for (int idx = tid; idx < (n + R) * DV; idx += kSThreads) {
            const int m = idx / DV, i = idx % DV;
            UU[idx] = m < n ? a.buf_u[((size_t)bh * W + m) * DV + i] : a.comp_u[((size_t)bh * R + (m - n)) * DV + i];
        }
        // start: the old compensators' k~_c, then start vectors
        for (int idx = tid; idx < DK * P; idx += kSThreads) {
            const int j = idx / P, c = idx % P;
            // the old k~_c plus a small start-vector part, so that a zero
            // compensator (after the zero state) still gives a basis vector
            sm.X[j * kMaxP + c] = c < R ? fmaf(1e-3f, start_entry(j, c, DK), a.comp_val[((size_t)bh * R + c) * DK + j])
                                        : start_entry(j, c, DK);
        }
        cta_sync();
        // S_ij = sigma_i Q_ij c_j e^{L_n,j} + sum_m U[m][i] K^[m][j]
        constexpr int TPR = kSThreads / DV;  // threads per row
        constexpr int CPT = DK / TPR;        // columns per thread
        const int i = tid / TPR, jb = (tid % TPR) * CPT;
        const float sg = BF16S ? 1.0f : a.row_scale[(size_t)bh * DV + i];
        for (int j4 = 0; j4 < CPT; j4 += 4) {
            const int j = jb + j4;
            float x[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int jj = j + e;
                float q;
                if constexpr (BF16S) {
                    const uint16_t b = reinterpret_cast<const uint16_t *>(codes)[(size_t)i * DK + jj];
                    q = __uint_as_float((uint32_t)b << 16);
                } else if constexpr (PACK4) {
                    const int g = jj / 8, b = jj % 8;
                    const uint8_t byte = (uint8_t)codes[(size_t)i * CRB + 4 * g + (b & 3)];
                    const int nib = b < 4 ? (byte & 0xF) : (byte >> 4);
                    q = (float)(nib >= 8 ? nib - 16 : nib);
                } else {
                    q = (float)codes[(size_t)i * CRB + jj];
                }
                const float cj = BF16S ? 1.0f : a.col_smooth[(size_t)bh * DK + jj];
                x[e] = (sg * q) * (cj * expf(Lg(n - 1, jj)));
            }
            for (int m = 0; m < n + R; ++m) {
                const float u = UU[m * DV + i];
                const float4 k4 = *reinterpret_cast<const float4 *>(&KH[m * DK + j]);
                x[0] = fmaf(u, k4.x, x[0]);
                x[1] = fmaf(u, k4.y, x[1]);
                x[2] = fmaf(u, k4.z, x[2]);
                x[3] = fmaf(u, k4.w, x[3]);
            }
            *reinterpret_cast<float4 *>(&sm.S[i * SP + j]) = make_float4(x[0], x[1], x[2], x[3]);
        }
    }
    cta_sync();

    // ---------------------------------------------------------------- 2. G = S^T S
    {
        constexpr int CB = DK / 8;           // column blocks of 8
        constexpr int NB = (DK / 4) * CB;    // 4 x 8 blocks
        for (int blk = tid; blk < NB; blk += kSThreads) {
            const int j0 = 4 * (blk / CB), k0 = 8 * (blk % CB);
            float acc[4][8];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 8; ++y) acc[x][y] = 0.0f;
            for (int i = 0; i < DV; ++i) {
                const float4 av = *reinterpret_cast<const float4 *>(&sm.S[i * SP + j0]);
                const float4 b0 = *reinterpret_cast<const float4 *>(&sm.S[i * SP + k0]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&sm.S[i * SP + k0 + 4]);
                const float ar[4] = {av.x, av.y, av.z, av.w};
                const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(ar[x], br[y], acc[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                *reinterpret_cast<float4 *>(&sm.G[(j0 + x) * SP + k0]) =
                    make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
                *reinterpret_cast<float4 *>(&sm.G[(j0 + x) * SP + k0 + 4]) =
                    make_float4(acc[x][4], acc[x][5], acc[x][6], acc[x][7]);
            }
        }
    }
    cta_sync();

    // ---------------------------------------------------------------- 3. subspace iteration
    auto gv = [&]() {  // X = G V
        for (int idx = tid; idx < DK * (P / 4); idx += kSThreads) {
            const int j = idx / (P / 4), c0 = 4 * (idx % (P / 4));
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < DK; ++k) {
                const float g = sm.G[j * SP + k];
                const float4 v = *reinterpret_cast<const float4 *>(&sm.V[k * kMaxP + c0]);
                acc.x = fmaf(g, v.x, acc.x);
                acc.y = fmaf(g, v.y, acc.y);
                acc.z = fmaf(g, v.z, acc.z);
                acc.w = fmaf(g, v.w, acc.w);
            }
            *reinterpret_cast<float4 *>(&sm.X[j * kMaxP + c0]) = acc;
        }
        cta_sync();
    };
    orthonormalise<DK>(sm.V, sm.X, sm.dot, P);
    for (int step = 0; step < kSteps; ++step) {
        gv();
        orthonormalise<DK>(sm.V, sm.X, sm.dot, P);
    }

    // ---------------------------------------------------------------- 4. Rayleigh-Ritz
    gv();  // X = G V
    for (int idx = tid; idx < P * P; idx += kSThreads) {
        const int x = idx / P, y = idx % P;
        double h = 0.0;
        for (int j = 0; j < DK; ++j) h = fma((double)sm.V[j * kMaxP + x], (double)sm.X[j * kMaxP + y], h);
        sm.H[x * kMaxP + y] = h;
        sm.Z[x * kMaxP + y] = x == y ? 1.0 : 0.0;
    }
    cta_sync();
    // symmetrise (H is symmetric up to rounding)
    for (int idx = tid; idx < P * P; idx += kSThreads) {
        const int x = idx / P, y = idx % P;
        if (x < y) {
            const double h = 0.5 * (sm.H[x * kMaxP + y] + sm.H[y * kMaxP + x]);
            sm.H[x * kMaxP + y] = h;
            sm.H[y * kMaxP + x] = h;
        }
    }
    cta_sync();
    // cyclic Jacobi, round-robin ordering: in round t, pair k joins the
    // players p(k) and p(P-1-k) of the circle (player 0 fixed, the others
    // rotated by t); the P/2 pairs of a round are disjoint
    for (int sweep = 0; sweep < kSweeps; ++sweep) {
        // stop once the off-diagonal part is at FP64 round-off of the diagonal
        if (warp == 0) {
            double off = 0.0, dia = 0.0;
            for (int idx = lane; idx < P * P; idx += 32) {
                const int x = idx / P, y = idx % P;
                const double h = sm.H[x * kMaxP + y];
                if (x == y) dia = fma(h, h, dia);
                else off = fma(h, h, off);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                off += __shfl_xor_sync(0xffffffffu, off, o);
                dia += __shfl_xor_sync(0xffffffffu, dia, o);
            }
            if (lane == 0) sm.jacobi_done = off <= 1e-30 * dia;
        }
        cta_sync();
        if (sm.jacobi_done) break;
        for (int t = 0; t < P - 1; ++t) {
            auto player = [&](int k) { return k == 0 ? 0 : 1 + (k - 1 + t) % (P - 1); };
            if (tid < P / 2) {
                int p = player(tid), q = player(P - 1 - tid);
                if (p > q) { const int s = p; p = q; q = s; }
                const double hpp = sm.H[p * kMaxP + p], hqq = sm.H[q * kMaxP + q], hpq = sm.H[p * kMaxP + q];
                double c = 1.0, s = 0.0;
                if (fabs(hpq) > 1e-300 * (fabs(hpp) + fabs(hqq)) && hpq != 0.0) {
                    // the rotation that zeroes H[p][q]
                    const double th = (hqq - hpp) / (2.0 * hpq);
                    const double tt = (th >= 0.0 ? 1.0 : -1.0) / (fabs(th) + sqrt(1.0 + th * th));
                    c = 1.0 / sqrt(1.0 + tt * tt);
                    s = tt * c;
                }
                sm.rc[tid] = c;
                sm.rs[tid] = s;
            }
            cta_sync();
            // H <- J^T H J and Z <- Z J, J the product of the round's rotations:
            // first the columns of H and Z, then the rows of H
            for (int idx = tid; idx < (P / 2) * P; idx += kSThreads) {
                const int k = idx / P, x = idx % P;
                int p = player(k), q = player(P - 1 - k);
                if (p > q) { const int s = p; p = q; q = s; }
                const double c = sm.rc[k], s = sm.rs[k];
                const double hp = sm.H[x * kMaxP + p], hq = sm.H[x * kMaxP + q];
                sm.H[x * kMaxP + p] = c * hp - s * hq;
                sm.H[x * kMaxP + q] = s * hp + c * hq;
                const double zp = sm.Z[x * kMaxP + p], zq = sm.Z[x * kMaxP + q];
                sm.Z[x * kMaxP + p] = c * zp - s * zq;
                sm.Z[x * kMaxP + q] = s * zp + c * zq;
            }
            cta_sync();
            for (int idx = tid; idx < (P / 2) * P; idx += kSThreads) {
                const int k = idx / P, y = idx % P;
                int p = player(k), q = player(P - 1 - k);
                if (p > q) { const int s = p; p = q; q = s; }
                const double c = sm.rc[k], s = sm.rs[k];
                const double hp = sm.H[p * kMaxP + y], hq = sm.H[q * kMaxP + y];
                sm.H[p * kMaxP + y] = c * hp - s * hq;
                sm.H[q * kMaxP + y] = s * hp + c * hq;
            }
            cta_sync();
        }
    }
    // the r largest eigenvalues (ties to the smaller index), one warp
    if (warp == 0) {
        double lam = lane < P ? sm.H[lane * kMaxP + lane] : -1.0;
        for (int c = 0; c < R; ++c) {
            double bv = lam;
            int bi = lane < P ? lane : kMaxP;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ov > bv || (ov == bv && oi < bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            if (lane == bi) lam = -2.0;
            if (lane == 0) sm.order[c] = bi;
        }
    }
    cta_sync();
    // k~_c = V z_c (normalised), the sign making its largest-magnitude entry positive
    for (int c = warp; c < R; c += kSWarps) {
        const int e = sm.order[c];
        float v[DK / 32];
        float nn = 0.0f;
#pragma unroll
        for (int t = 0; t < DK / 32; ++t) {
            const int j = lane + 32 * t;
            double x = 0.0;
            for (int k = 0; k < P; ++k) x = fma((double)sm.V[j * kMaxP + k], sm.Z[k * kMaxP + e], x);
            v[t] = (float)x;
            nn = fmaf(v[t], v[t], nn);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nn += __shfl_xor_sync(0xffffffffu, nn, o);
        const float inv = nn > 0.0f ? rsqrtf(nn) : 0.0f;
        // the first index of the largest magnitude decides the sign
        float best = -1.0f;
        int bj = DK;
#pragma unroll
        for (int t = 0; t < DK / 32; ++t) {
            v[t] *= inv;
            const float m = fabsf(v[t]);
            if (m > best) {
                best = m;
                bj = lane + 32 * t;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
            if (ob > best || (ob == best && oj < bj)) {
                best = ob;
                bj = oj;
            }
        }
        float sgn = 1.0f;
#pragma unroll
        for (int t = 0; t < DK / 32; ++t)
            if (lane + 32 * t == bj) sgn = v[t] < 0.0f ? -1.0f : 1.0f;
        sgn = __shfl_sync(0xffffffffu, sgn, bj % 32);
#pragma unroll
        for (int t = 0; t < DK / 32; ++t) sm.vc[c * DK + lane + 32 * t] = sgn * v[t];
    }
    cta_sync();
    // u_c = S k~_c (one warp per row group, lanes over the key channels)
    for (int idx = warp; idx < R * DV; idx += kSWarps) {
        const int c = idx / DV, i = idx % DV;
        float d = 0.0f;
        for (int j = lane; j < DK; j += 32) d = fmaf(sm.S[i * SP + j], sm.vc[c * DK + j], d);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) sm.uc[c * DV + i] = d;
    }
    cta_sync();

    // ---------------------------------------------------------------- 5. residual, C3-C4
    float *comp_val = a.comp_val + (size_t)bh * R * DK;
    float *comp_u = a.comp_u + (size_t)bh * R * DV;
    for (int idx = tid; idx < R * DK; idx += kSThreads) comp_val[idx] = sm.vc[idx];
    for (int idx = tid; idx < R * DV; idx += kSThreads) comp_u[idx] = sm.uc[idx];
    for (int idx = tid; idx < R; idx += kSThreads) a.comp_row[(size_t)bh * R + idx] = 0;
    const int c0 = T::col0(lane);
    float Sreg[T::NR][4];
#pragma unroll
    for (int nn = 0; nn < T::NR; ++nn) {
        const int i = T::row(warp, lane, nn);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float x = sm.S[i * SP + c0 + e];
            for (int c = 0; c < R; ++c) x = fmaf(-sm.uc[c * DV + i], sm.vc[c * DK + c0 + e], x);
            Sreg[nn][e] = x;
        }
    }
    SnapPtr out{a.codes + (size_t)bh * DV * CRB, a.row_scale + (size_t)bh * DV,
                a.col_smooth + (size_t)bh * DK, nullptr, nullptr};
    quantize_tile<DK, DV, kSWarps>(Sreg, 0, a.smoothing != 0, a.bits, sm.q, out);
}

template <int DK, int DV, int GATE, int FMT>
cudaError_t launch_s(const SvdArgs &A, int grid, cudaStream_t stream) {
    static_assert(svd_smem_bytes<DK, DV>() <= 227 * 1024, "shared memory of the SVD rule");
    auto kern = svd_kernel<DK, DV, GATE, FMT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)svd_smem_bytes<DK, DV>());
    if (e != cudaSuccess) return e;
    kern<<<grid, kSThreads, svd_smem_bytes<DK, DV>(), stream>>>(A);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_sg(const SvdArgs &A, int gate, int grid, cudaStream_t stream) {
    const int fmt = code_format(A.d.bits);
    if (gate == 1) {
        if (fmt == kCodesI4) return launch_s<DK, DV, 1, kCodesI4>(A, grid, stream);
        if (fmt == kCodesBF16) return launch_s<DK, DV, 1, kCodesBF16>(A, grid, stream);
        return launch_s<DK, DV, 1, kCodesI8>(A, grid, stream);
    }
    if (fmt == kCodesI4) return launch_s<DK, DV, 0, kCodesI4>(A, grid, stream);
    if (fmt == kCodesBF16) return launch_s<DK, DV, 0, kCodesBF16>(A, grid, stream);
    return launch_s<DK, DV, 0, kCodesI8>(A, grid, stream);
}

cudaError_t launch_svd(const SvdArgs &A, int d_k, int d_v, int gate, cudaStream_t stream) {
    if (A.d.R < 1 || A.d.R > kMaxComp || A.d.R > d_k || !A.d.comp_u) return cudaErrorInvalidValue;
    if (A.S == nullptr && (A.d.pos < 1 || A.d.pos > kMaxRec)) return cudaErrorInvalidValue;
    const int grid = A.d.B * A.d.H;
    if (d_k == 128 && d_v == 128) return launch_sg<128, 128>(A, gate, grid, stream);
    if (d_k == 128 && d_v == 64) return launch_sg<128, 64>(A, gate, grid, stream);
    if (d_k == 64 && d_v == 128) return launch_sg<64, 128>(A, gate, grid, stream);
    if (d_k == 64 && d_v == 64) return launch_sg<64, 64>(A, gate, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_svd_quantize(const QuantArgs &q, int d_k, int d_v, cudaStream_t stream) {
    SvdArgs A{};
    A.S = q.S;
    DecodeArgs &d = A.d;
    d.codes = q.codes;
    d.row_scale = q.row_scale;
    d.col_smooth = q.col_smooth;
    d.comp_row = q.comp_row;
    d.comp_val = q.comp_val;
    d.comp_u = q.comp_u;
    d.B = q.BH;
    d.H = 1;
    d.R = q.R;
    d.W = 1;
    d.smoothing = q.smoothing;
    d.bits = q.bits;
    if (!q.S) return cudaErrorInvalidValue;  // the zero state: see launch_quantize
    return launch_svd(A, d_k, d_v, 0, stream);
}

cudaError_t launch_svd_commit(const DecodeArgs &a, int d_k, int d_v, int gate, cudaStream_t stream) {
    SvdArgs A{};
    A.S = nullptr;
    A.d = a;
    return launch_svd(A, d_k, d_v, gate, stream);
}

}  // namespace lq
