// lq_kernels.h -- internal interface between the C-ABI layer (lq_api.cu) and
// the kernel launchers.  Not installed; not part of the ABI.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace lq {

// Storage of a snapshot's residual: integer codes one per byte (8- and 6-bit
// widths), two per byte (4-bit), or BF16 values (bits = 16).
enum CodeFormat { kCodesI8 = 0, kCodesI4 = 1, kCodesBF16 = 2 };
__host__ __device__ constexpr int code_format(int bits) {
    return bits == 4 ? kCodesI4 : bits == 16 ? kCodesBF16 : kCodesI8;
}
// Bytes of one value row of the residual with d_k key channels.
__host__ __device__ constexpr int code_row_bytes(int fmt, int dk) {
    return fmt == kCodesI4 ? dk / 2 : fmt == kCodesBF16 ? 2 * dk : dk;
}

// cuTensorMapEncodeTiled of the driver, looked up once (nullptr when the
// driver does not provide it).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// Arguments of the decode and commit kernels.
struct DecodeArgs {
    int8_t *codes;
    float *row_scale;
    float *col_smooth;
    int32_t *comp_row;
    float *comp_val;
    float *comp_u;  // SVD compensator rule: u_c [BH][R][DV]; nullptr for the row rule
    float *buf_gate;
    float *buf_k;
    float *buf_u;
    const void *q;
    const void *k;
    const void *v;
    const float *alpha;
    const float *beta;
    void *o;
    int B, H, W, R;
    int delta;    // 1: b_t = D_t k_t (delta rule); 0: b_t = 0
    int pos;      // records already buffered (the same for every sequence)
    int n_steps;  // tokens decoded by this launch (0: commit only)
    int smoothing;
    int bits;     // code width: 8 or 6 (one code per byte), 4 (two per byte), 16 (BF16)
    // per-sequence window positions [B] (device), or nullptr.  When set, the
    // decode takes one token per sequence b with seq_pos[b] in [0, W) at
    // window position seq_pos[b] + 1 (pos and n_steps are then W - 1 and 1,
    // the sizes the stages are laid out for) and skips sequences with
    // seq_pos[b] < 0; the commit takes the sequences with seq_pos[b] == W - 1
    // (pos is then W).
    const int32_t *seq_pos;
    // with seq_pos set, the commit takes the sequences whose seq_pos equals
    // commit_match (W - 1 after a ragged decode; p, with pos = p, when the
    // open windows of p records are flushed)
    int commit_match;
};

// Arguments of the quantize-from-FP32 kernel (init, prefill snapshots).
struct QuantArgs {
    const float *S;  // [BH][DV][DK], nullptr = zeros
    int8_t *codes;
    float *row_scale;
    float *col_smooth;
    int32_t *comp_row;
    float *comp_val;
    float *comp_u;  // SVD compensator rule: u_c [BH][R][DV]; nullptr for the row rule
    int BH, R, smoothing;
    int bits;  // code width: 8 or 6 (one code per byte), 4 (two per byte), 16 (BF16)
};

// Arguments of the FP32-state recurrence kernel (prefill, FP32 per-step).
struct RecurArgs {
    float *S;  // [BH][DV][DK] in/out
    const void *q;
    const void *k;
    const void *v;
    const float *alpha;
    const float *beta;
    void *o;
    int B, H;
    int delta;    // 1: b_t = D_t k_t (delta rule); 0: b_t = 0
    int T_total;  // tokens in the activation tensors (time stride)
    int t0, nt;   // tokens [t0, t0+nt) processed by this launch
};

// Arguments of the chunked prefill (lq_chunk.cu): one pass of nc chunks of
// 64 tokens starting at token t0 of every sequence.
struct ChunkArgs {
    float *S;            // [BH][DV][128] FP32 state, in/out
    const float *alpha;  // [B][T_total][H]
    const float *beta;   // [B][T_total][H]
    void *o;             // BF16 [B][T_total][H][DV]
    float *ws;           // workspace [nc][BH] blocks of 48 KB ([PT; T] of each chunk as
                         // three BF16 parts in the tensor-core operand layout)
    int B, H, DV, T_total, t0, nc, delta;
};

// Workspace bytes of a pass of `chunks` chunks over BH heads.
size_t chunk_workspace_bytes(int BH, int chunks);

// Whether the tensor-core chunked prefill covers this shape (scalar gate,
// BF16 io, d_k = 128, d_v in {64, 128}).
bool chunk_path_supported(int d_k, int d_v, int gate, bool bf16);

// One pass in two launches: the [PT; T] preparation of every chunk into
// a.ws (reads q, k, alpha, beta), then the chunks in order (reads a.ws, q, k,
// v, alpha, beta and the state; writes the outputs and the state).
cudaError_t launch_chunk_prep(const ChunkArgs &a, const void *q, const void *k, cudaStream_t stream);
cudaError_t launch_chunk_scan(const ChunkArgs &a, const void *q, const void *k, const void *v,
                              cudaStream_t stream);

// Decodes a.n_steps >= 1 tokens (records a.pos .. a.pos + n_steps - 1).
cudaError_t launch_decode(const DecodeArgs &a, int d_k, int d_v, int gate, bool bf16,
                          cudaStream_t stream);

// Commits the window of a.pos >= 1 buffered records (a.n_steps unused):
// rebuild, compensators, smoothing, codes, written over the snapshot.
cudaError_t launch_commit(const DecodeArgs &a, int d_k, int d_v, int gate, cudaStream_t stream);

// seq_pos[b] <- (seq_pos[b] + 1) mod W for the sequences with 0 <= seq_pos[b] < W.
cudaError_t launch_advance_positions(int32_t *seq_pos, int B, int W, cudaStream_t stream);

// seq_pos[b] <- 0 for the sequences with 0 < seq_pos[b] < W (after their
// windows were committed); a position >= W sets the device error word.
cudaError_t launch_reset_positions(int32_t *seq_pos, int B, int W, cudaStream_t stream);

// Reads the device error word and clears it (synchronizes the device).
cudaError_t read_and_clear_dev_error(unsigned int *out);

// Quantizes FP32 states (a.S) into snapshots; with a.comp_u set, by the SVD
// compensator rule (lq_svd.cu).
cudaError_t launch_quantize(const QuantArgs &a, int d_k, int d_v, cudaStream_t stream);

// The SVD compensator rule (lq_svd.cu): snapshots of FP32 states (a.S), and
// the window commit of a.pos >= 1 records (rebuild from the snapshot and the
// records, then the rule), written over the snapshot.
cudaError_t launch_svd_quantize(const QuantArgs &a, int d_k, int d_v, cudaStream_t stream);
cudaError_t launch_svd_commit(const DecodeArgs &a, int d_k, int d_v, int gate, cudaStream_t stream);

// rows_per_cta selects the parallelisation: the full head (one CTA per head,
// for a few tokens) or a slice of rows (many CTAs per head, for long runs).
cudaError_t launch_recurrence(const RecurArgs &a, int d_k, int d_v, int gate, bool bf16,
                              bool long_run, cudaStream_t stream);

}  // namespace lq
