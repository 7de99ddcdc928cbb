// lq_quant.cuh -- the register tile of one head's state and the commit
// quantizer on it: Compensator Tokens, residual smoothing, per-row int8.
//
// "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
// Quantization", Abstract and Figure 4: the state's largest outliers are kept
// as a few high-precision Compensator Tokens (flattening the residual's row
// l2 norms), the residual is smoothed across channels and quantized once to
// 8 bits.  The pages fix neither rule; this library's rule is:
//   C2  the r rows of largest l2 norm become compensators (largest first, an
//       exact tie to the smaller row), stored exactly in FP32, and are zeroed
//       in the residual R;
//   C3  c_j = sqrt(max_i |R_ij|) (1 for a zero column or with smoothing off),
//       R'_ij = R_ij / c_j;
//   C4  sigma_i = max_j |R'_ij| / q (stored),
//       Q_ij = rne(R'_ij / sigma_i) in [-q, q], Q = 0 where sigma_i = 0,
//       with q = 2^(bits-1) - 1: 127 for 8-bit codes, 31 and 7 for the 6- and
//       4-bit widths of the paper's lower-precision groups (Table 1); 4-bit
//       codes are stored two per byte (low nibble: channel 8g+b, high
//       nibble: channel 8g+4+b, in byte 4g+b of a row).
// bits = 16 is the paper's BF16 state (Table 2): C2 as above, then c = 1,
// sigma = 1 and the residual itself rounded to BF16 (nearest, ties to even).
// Every division and square root is one IEEE round-to-nearest FP32 operation
// (__fdiv_rn, __fsqrt_rn), so the codes of a given FP32 state are exactly
// determined.  (The window commit, lq_commit.cu, multiplies by the FP32
// inverses instead: one more rounding, codes within one step of these.)
#pragma once

#include "lq_common.cuh"

namespace lq {

constexpr int kMaxComp = 16;

// Ownership of a d_v x d_k state by a CTA of NWARPS warps.  Each lane owns 4
// consecutive key channels (columns) of NR rows: LPR lanes cover one row, a
// warp instruction covers RPI rows, warp w owns rows [w*RPW, (w+1)*RPW).
template <int DK, int DV, int NWARPS>
struct Tile {
    static constexpr int LPR = DK / 4;
    static constexpr int RPI = 32 / LPR;
    static constexpr int RPW = DV / NWARPS;
    static constexpr int NR = RPW / RPI;
    static constexpr int NTHREADS = NWARPS * 32;
    static_assert(DK == 64 || DK == 128, "d_k must be 64 or 128");
    static_assert(RPW % RPI == 0 && NR >= 1, "tile does not divide the state");
    __device__ static int col0(int lane) { return 4 * (lane % LPR); }
    __device__ static int row(int warp, int lane, int n) {
        return warp * RPW + n * RPI + lane / LPR;
    }
};

// Device pointers of one head's snapshot.
struct SnapPtr {
    int8_t *codes;      // [DV][DK], [DV][DK/2] bytes of packed 4-bit codes, or BF16 [DV][DK]
    float *row_scale;   // [DV]
    float *col_smooth;  // [DK]
    int32_t *comp_row;  // [R]
    float *comp_val;    // [R][DK]
};

// Shared scratch of the quantizer.  colpart rows are written with 16-byte
// vector stores, so the struct and that member are 16-byte aligned.
template <int DK, int DV, int NWARPS>
struct alignas(16) QuantSmem {
    float rowss[DV];
    int comp_idx[DV];
    alignas(16) float colpart[NWARPS * Tile<DK, DV, NWARPS>::RPI][DK];
    float cs[DK];
    int sel[kMaxComp];
};

// C2-C4 on the register tile S (the FP32 state of one head, owned as Tile
// describes), writing the snapshot to `out` with codes of width `bits` (8, 6
// or 4; 16 = BF16 residual).  The NWARPS*32 threads that own the tile
// (threads 0 .. NWARPS*32-1) call it; it synchronises them on named barrier 1.
template <int DK, int DV, int NWARPS>
__device__ __forceinline__ void quantize_tile(float (&S)[Tile<DK, DV, NWARPS>::NR][4], int R,
                                              bool smoothing, int bits,
                                              QuantSmem<DK, DV, NWARPS> &sm, const SnapPtr &out) {
    using T = Tile<DK, DV, NWARPS>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = T::col0(lane);

    const int gbase = lane & ~(T::LPR - 1);  // first lane of this lane's row group
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const bool pack4 = bits == 4, bf16s = bits == 16;
    if (bf16s) smoothing = false;  // c = 1 for the BF16 residual
    // C2 (1/2): squared row norms (order-preserving for the selection),
    // reduced across the row's lanes with a transposing reduction
    {
        float ss[T::NR];
#pragma unroll
        for (int n = 0; n < T::NR; ++n) {
            ss[n] = S[n][0] * S[n][0];
            ss[n] = fmaf(S[n][1], S[n][1], ss[n]);
            ss[n] = fmaf(S[n][2], S[n][2], ss[n]);
            ss[n] = fmaf(S[n][3], S[n][3], ss[n]);
        }
        transposed_sum<T::NR, T::LPR>(ss, lane);
        const int n = transposed_index<T::NR, T::LPR>(lane);
        if ((lane & (T::LPR - 1)) == transposed_owner<T::NR, T::LPR>(n))
            sm.rowss[T::row(warp, lane, n)] = ss[0];
    }
    for (int i = tid; i < DV; i += T::NTHREADS) sm.comp_idx[i] = -1;
    consumer_sync<T::NTHREADS>();

    // C2 (2/2): warp 0 selects the R largest, ties to the smaller row
    if (warp == 0 && R > 0) {
        constexpr int PER = DV / 32;
        float val[PER];
#pragma unroll
        for (int p = 0; p < PER; ++p) val[p] = sm.rowss[lane + 32 * p];
        for (int c = 0; c < R; ++c) {
            float bv = -1.0f;
            int bi = DV;
#pragma unroll
            for (int p = 0; p < PER; ++p)
                if (val[p] > bv) {
                    bv = val[p];
                    bi = lane + 32 * p;
                }
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, s);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, s);
                if (ov > bv || (ov == bv && oi < bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
#pragma unroll
            for (int p = 0; p < PER; ++p)
                if (lane + 32 * p == bi) val[p] = -1.0f;
            if (lane == 0) {
                sm.sel[c] = bi;
                sm.comp_idx[bi] = c;
            }
        }
    }
    consumer_sync<T::NTHREADS>();

    // Compensator rows leave the residual, exactly
#pragma unroll
    for (int n = 0; n < T::NR; ++n) {
        const int c = sm.comp_idx[T::row(warp, lane, n)];
        if (c >= 0) {
            *reinterpret_cast<float4 *>(out.comp_val + (size_t)c * DK + c0) =
                make_float4(S[n][0], S[n][1], S[n][2], S[n][3]);
            S[n][0] = S[n][1] = S[n][2] = S[n][3] = 0.0f;
        }
    }
    if (tid < R) out.comp_row[tid] = sm.sel[tid];

    // C3: smoothing factor per key channel
    {
        float cm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int n = 0; n < T::NR; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) cm[e] = fmaxf(cm[e], fabsf(S[n][e]));
        *reinterpret_cast<float4 *>(&sm.colpart[warp * T::RPI + lane / T::LPR][c0]) =
            make_float4(cm[0], cm[1], cm[2], cm[3]);
    }
    consumer_sync<T::NTHREADS>();
    for (int j = tid; j < DK; j += T::NTHREADS) {
        float m = 0.0f;
#pragma unroll 4
        for (int p = 0; p < NWARPS * T::RPI; ++p) m = fmaxf(m, sm.colpart[p][j]);
        const float c = (smoothing && m > 0.0f) ? __fsqrt_rn(m) : 1.0f;
        out.col_smooth[j] = c;
        sm.cs[j] = c;
    }
    consumer_sync<T::NTHREADS>();
    float cj[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) cj[e] = sm.cs[c0 + e];

    // C4: per-row scale and codes of R' = R / c.  Row maxima are reduced with
    // a transposing reduction; each row's scale is computed once, by the lane
    // that holds the row's maximum, and broadcast.
    float sig_own;
    {
        float mx[T::NR];
#pragma unroll
        for (int n = 0; n < T::NR; ++n) {
            mx[n] = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                S[n][e] = __fdiv_rn(S[n][e], cj[e]);
                mx[n] = fmaxf(mx[n], fabsf(S[n][e]));
            }
        }
        transposed_max<T::NR, T::LPR>(mx, lane);
        const int n = transposed_index<T::NR, T::LPR>(lane);
        sig_own = __fdiv_rn(mx[0], qmax);
        if ((lane & (T::LPR - 1)) == transposed_owner<T::NR, T::LPR>(n))
            out.row_scale[T::row(warp, lane, n)] = bf16s ? 1.0f : sig_own;
    }
#pragma unroll
    for (int n = 0; n < T::NR; ++n) {
        const float sig =
            __shfl_sync(0xffffffffu, sig_own, gbase + transposed_owner<T::NR, T::LPR>(n));
        const int row = T::row(warp, lane, n);
        if (bf16s) {
            // the residual itself, rounded to BF16 (c = 1, so S is unscaled)
            const __nv_bfloat162 p0 = __floats2bfloat162_rn(S[n][0], S[n][1]);
            const __nv_bfloat162 p1 = __floats2bfloat162_rn(S[n][2], S[n][3]);
            *reinterpret_cast<uint2 *>(out.codes + ((size_t)row * DK + c0) * 2) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&p0),
                           *reinterpret_cast<const uint32_t *>(&p1));
            continue;
        }
        // round half to even by the magic-number addition (|y| <= q here),
        // clamp, and pack the four low bytes
        int iv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // Q = 0 where sigma = 0 (a zero row, or a maximum below q times
            // the smallest FP32 value)
            const float y = sig > 0.0f ? fminf(fmaxf(__fdiv_rn(S[n][e], sig), -qmax), qmax) : 0.0f;
            iv[e] = __float_as_int(__fadd_rn(y, 12582912.0f)) - 0x4B400000;
        }
        const uint32_t packed = __byte_perm(__byte_perm(iv[0], iv[1], 0x0040),
                                            __byte_perm(iv[2], iv[3], 0x0040), 0x5410);
        if (pack4) {
            // two's-complement nibbles; lanes 2p and 2p+1 of a row hold the
            // channels 8g..8g+3 and 8g+4..8g+7 of one 8-channel group
            const uint32_t nib = packed & 0x0F0F0F0Fu;
            const uint32_t hi = __shfl_xor_sync(0xffffffffu, nib, 1);
            if ((c0 & 4) == 0)
                *reinterpret_cast<uint32_t *>(out.codes + (size_t)row * (DK / 2) + c0 / 2) =
                    nib | (hi << 4);
        } else {
            *reinterpret_cast<uint32_t *>(out.codes + (size_t)row * DK + c0) = packed;
        }
    }
}

}  // namespace lq
