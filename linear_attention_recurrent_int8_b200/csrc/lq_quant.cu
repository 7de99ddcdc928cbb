// lq_quant.cu -- quantization of FP32 states into snapshots: state
// initialisation and the prefill's prefix-cache snapshots ("LeapQuant:
// Efficient Linear Attention with Accurate Recurrent State Quantization",
// Figure 1(b): one state per 1,024 cached tokens).  One CTA per head loads the
// FP32 state into the register tile with coalesced 16-byte loads and runs the
// commit quantizer on it (lq_quant.cuh).
#include "lq_kernels.h"
#include "lq_quant.cuh"

namespace lq {
namespace {

constexpr int kWarps = 8;

template <int DK, int DV>
__global__ void __launch_bounds__(kWarps * 32) quantize_kernel(const QuantArgs a) {
    using T = Tile<DK, DV, kWarps>;
    __shared__ QuantSmem<DK, DV, kWarps> qsm;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int c0 = T::col0(lane);
    float S[T::NR][4];
#pragma unroll
    for (int n = 0; n < T::NR; ++n) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.S)
            x = *reinterpret_cast<const float4 *>(a.S + ((size_t)bh * DV + T::row(warp, lane, n)) * DK +
                                                  c0);
        S[n][0] = x.x;
        S[n][1] = x.y;
        S[n][2] = x.z;
        S[n][3] = x.w;
    }
    const size_t code_bytes = (size_t)DV * code_row_bytes(code_format(a.bits), DK);
    SnapPtr out{a.codes + (size_t)bh * code_bytes, a.row_scale + (size_t)bh * DV,
                a.col_smooth + (size_t)bh * DK, a.comp_row ? a.comp_row + (size_t)bh * a.R : nullptr,
                a.comp_val ? a.comp_val + (size_t)bh * a.R * DK : nullptr};
    quantize_tile<DK, DV, kWarps>(S, a.R, a.smoothing != 0, a.bits, qsm, out);
}

template <int DK, int DV>
cudaError_t launch_q(const QuantArgs &a, cudaStream_t stream) {
    quantize_kernel<DK, DV><<<a.BH, kWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs &a, int d_k, int d_v, cudaStream_t stream) {
    if (a.comp_u && a.R > 0) {
        if (a.S) return launch_svd_quantize(a, d_k, d_v, stream);
        // the zero state under the SVD rule: every u_c = 0, and the row
        // rule's kernel writes the zero residual (codes, sigma = 0, c = 1)
        // and zero k~_c
        const cudaError_t e = cudaMemsetAsync(a.comp_u, 0, (size_t)a.BH * a.R * d_v * sizeof(float), stream);
        if (e != cudaSuccess) return e;
    }
    if (d_k == 128 && d_v == 128) return launch_q<128, 128>(a, stream);
    if (d_k == 128 && d_v == 64) return launch_q<128, 64>(a, stream);
    if (d_k == 64 && d_v == 128) return launch_q<64, 128>(a, stream);
    if (d_k == 64 && d_v == 64) return launch_q<64, 64>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace lq
