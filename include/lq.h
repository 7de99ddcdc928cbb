/*
 * lq.h -- C ABI of liblq: int8 per-window recurrent-state decode for
 * delta-rule linear attention (Gated DeltaNet scalar gate, Kimi-Delta-
 * Attention per-channel gate) on NVIDIA B200 (sm_100a).
 *
 * The method is LeapQuant ("LeapQuant: Efficient Linear Attention with
 * Accurate Recurrent State Quantization", Abstract and Figure 2): the int8
 * boundary state S^_0 stays fixed for a window of W tokens, the window's
 * updates are buffered in FP32, every output o_t = S_t q_t is computed from
 * S^_0 plus the buffer, and at the window end the state is rebuilt, its
 * largest rows are kept as FP32 Compensator Tokens (Figure 4), the residual is
 * smoothed across key channels and re-quantized once to int8.
 *
 * Recurrence (equation 1 of the paper, whose instances are its Appendix
 * Table 4):  S_t = S_{t-1} D_t + (v_t - S_{t-1} b_t) k~_t^T,  o_t = S_t q_t,
 * with S in R^{d_v x d_k} (row = value channel), k~_t = beta_t k_t and
 *   scalar gate (Gated DeltaNet, Table 4):   D_t = alpha_t I,       b_t = alpha_t k_t
 *   diagonal gate (Kimi Delta Attention):    D_t = Diag(alpha_t),   b_t = alpha_t * k_t
 * and, with lq_config.delta = 0, b_t = 0 for either gate (the Table 4 rows of
 * linear attention, RetNet, Mamba2 and GLA; k~_t = beta_t k_t, so those rows'
 * k~ = k is beta = 1).
 *
 * Conventions of every call:
 *  - Every pointer argument named as device memory is caller-owned CUDA
 *    device memory (for example a torch tensor's data_ptr()).  The library
 *    allocates no device memory and keeps no pointer after a call returns,
 *    except the ones the caller stores in lq_state.
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *    They never synchronize, except lq_device_errors.
 *  - Arguments are validated before anything is launched.  A call that
 *    returns an error status other than LQ_ERR_CUDA has launched nothing and
 *    changed nothing (lq_decode_window and lq_decode_ragged state their
 *    LQ_ERR_CUDA cases).
 *  - A launch failure reported by the CUDA runtime returns LQ_ERR_CUDA.
 *  - No C++ exception crosses this boundary.
 *  - One lq_state is used by one stream at a time.
 *  - Layouts are row-major.  B = batch, H = heads, n = tokens of the call.
 *      activations  q, k: [B, n, H, d_k] (16B)   v: [B, n, H, d_v] (16B)
 *                   o: [B, n, H, d_v] (aligned to its element)
 *                   alpha: [B, n, H] (scalar gate) or [B, n, H, d_k] (diagonal, (16B))
 *                   beta:  [B, n, H]                       (all FP32)
 *      q, k, v, o are FP32 or BF16 (lq_config.io_dtype).
 *  - Pointers marked (16B) must be 16-byte aligned (LQ_ERR_MISALIGNED).
 */
#ifndef LQ_H
#define LQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LQ_API __attribute__((visibility("default")))
#else
#define LQ_API
#endif

/* Same type as cudaStream_t, so the header needs no CUDA include. */
typedef struct CUstream_st *lq_stream_t;

typedef enum {
    LQ_OK = 0,
    LQ_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size or enum value    */
    LQ_ERR_UNSUPPORTED = 2,      /* valid but not built: d_k, d_v not in {64,128} */
    LQ_ERR_WINDOW_FULL = 3,      /* pos + n_steps > W                       */
    LQ_ERR_WINDOW_OPEN = 4,      /* the call needs pos == 0                  */
    LQ_ERR_MISALIGNED = 5,       /* a (16B) pointer is not 16-byte aligned   */
    LQ_ERR_CUDA = 6              /* the CUDA runtime reported an error       */
} lq_status;

typedef enum { LQ_GATE_SCALAR = 0, LQ_GATE_DIAG = 1 } lq_gate;
typedef enum { LQ_F32 = 0, LQ_BF16 = 1 } lq_dtype;

/* How the r Compensator Tokens of a snapshot are chosen ("LeapQuant: ...",
 * Abstract and Figure 4 keep the state's largest outliers in high precision
 * and flatten the residual's row norms, without fixing the rule):
 *   LQ_COMP_ROWS  the r value rows of largest l2 norm, stored exactly
 *                 (comp_row, comp_val);
 *   LQ_COMP_SVD   the r largest singular triplets of the FP32 state, as
 *                 rank-one terms u_c k~_c^T with u_c = s_c U_c (comp_u) and
 *                 k~_c = V_c (comp_val), the largest-magnitude entry of k~_c
 *                 positive; the residual S - sum_c u_c k~_c^T is smoothed
 *                 and quantized as with LQ_COMP_ROWS.  This library's variant:
 *                 the pages fix no rule, and the singular triplets are
 *                 computed by subspace iteration (see lq_state_init). */
typedef enum { LQ_COMP_ROWS = 0, LQ_COMP_SVD = 1 } lq_comp_rule;

typedef struct {
    int32_t batch;       /* B >= 1                                          */
    int32_t heads;       /* H >= 1; B * H <= 2^24 (LQ_ERR_INVALID_ARGUMENT)  */
    int32_t d_k;         /* 64 or 128                                       */
    int32_t d_v;         /* 64 or 128                                       */
    int32_t window;      /* W in [1, 32]: tokens per quantization window    */
    int32_t n_comp;      /* r in [0, 16], r <= d_v: Compensator Tokens      */
    int32_t gate;        /* lq_gate                                         */
    int32_t io_dtype;    /* lq_dtype of q, k, v, o                          */
    int32_t smoothing;   /* 1: residual smoothing on; 0: c == 1             */
    int32_t auto_commit; /* 1: the decode call that fills the window also
                            commits it (a second launch)                    */
    int32_t delta;       /* 1: delta rule, b_t = D_t k_t (Gated DeltaNet,
                            DeltaNet with alpha = 1, Kimi Delta Attention);
                            0: b_t = 0, u_t = v_t (linear attention, RetNet,
                            Mamba2, GLA: the b = 0 rows of Table 4)         */
    int32_t bits;        /* code width of the snapshot: 8 (0 also means 8), 6
                            or 4.  Codes lie in [-q, q], q = 2^(bits-1) - 1
                            (127, 31, 7); the paper reports 8-, 6- and 4-bit
                            state groups (Table 1) and fixes no format, so
                            the narrower widths are this library's variant of
                            the same quantizer.  8 and 6 store one code per
                            byte, 4 stores two (see lq_snapshot).
                            16: the BF16 state of the paper's Table 2
                            ablation: compensators as above, the residual
                            stored as BF16 values (round to nearest even),
                            no smoothing, row_scale = col_smooth = 1.      */
    int32_t comp_rule;   /* lq_comp_rule (0 = LQ_COMP_ROWS)                  */
} lq_config;

/* The quantized boundary state of every (b, h), all device memory:
 *   codes      int8    [B*H][d_v][d_k]  (16B)  Q, residual codes in [-q, q]
 *                                              (bits 8 or 6);
 *              uint8   [B*H][d_v][d_k/2] (16B) at bits = 4: in each group of
 *                                              8 key channels 8g..8g+7 of a
 *                                              row, byte 4g+b (b = 0..3) holds
 *                                              channel 8g+b in its low nibble
 *                                              and 8g+4+b in its high nibble,
 *                                              both two's complement;
 *              bf16    [B*H][d_v][d_k]  (16B)  at bits = 16: the residual
 *   row_scale  float   [B*H][d_v]       (16B)  sigma_i (0 for a zero row)
 *   col_smooth float   [B*H][d_k]       (16B)  c_j (1 when smoothing is off)
 *   comp_row   int32   [B*H][r]                row index of each compensator,
 *                                              largest l2 norm first
 *   comp_val   float   [B*H][r][d_k]    (16B)  the compensator rows (FP32)
 *   comp_u     float   [B*H][r][d_v]    (16B)  LQ_COMP_SVD: u_c = s_c U_c
 * S^_0 = Diag(row_scale) codes Diag(col_smooth) + sum_c e_{comp_row[c]} comp_val[c]^T
 * (LQ_COMP_ROWS), or + sum_c comp_u[c] comp_val[c]^T (LQ_COMP_SVD; comp_row
 * then holds zeros).  comp_row, comp_val and comp_u may be NULL when r == 0. */
typedef struct {
    int8_t *codes;
    float *row_scale;
    float *col_smooth;
    int32_t *comp_row;
    float *comp_val;
    float *comp_u;   /* LQ_COMP_SVD only (else ignored, may be NULL)      */
} lq_snapshot;

/* A decode state.  The caller fills `snap` and the three window buffers with
 * device pointers before lq_state_init; the library fills `cfg` and `pos`.
 *   buf_gate float [B*H][W][1 or d_k] (16B) running log gate L_t = sum log alpha
 *   buf_k    float [B*H][W][d_k]      (16B) k~_t = beta_t k_t
 *   buf_u    float [B*H][W][d_v]      (16B) u_t = v_t - S_{t-1} b_t
 * `pos` counts the tokens buffered in the open window (the same for every
 * sequence of the batch), or is LQ_POS_PER_SEQUENCE once lq_decode_ragged has
 * run: the window positions then live on the device (its seq_pos array) and
 * the calls that need every window closed (lq_decode_window,
 * lq_window_commit, lq_prefill_chunk, lq_state_snapshot, lq_state_restore)
 * return LQ_ERR_WINDOW_OPEN until lq_ragged_flush (or lq_state_init) returns
 * pos to 0.  `impl` is reserved (NULL). */
/* lq_state.pos after lq_decode_ragged: per-sequence window positions. */
#define LQ_POS_PER_SEQUENCE (-1)

typedef struct {
    lq_config cfg;
    lq_snapshot snap;
    float *buf_gate;
    float *buf_k;
    float *buf_u;
    int32_t pos;
    void *impl;
} lq_state;

/* Number of elements of one buffer of a state with configuration `cfg`
 * (for sizing allocations; codes count elements of their storage type:
 * int8, uint8 at bits = 4, bf16 at bits = 16); -1 for an invalid
 * configuration.
 * which: 0 codes, 1 row_scale, 2 col_smooth, 3 comp_row, 4 comp_val,
 *        5 buf_gate, 6 buf_k, 7 buf_u, 8 comp_u (0 with LQ_COMP_ROWS). */
LQ_API int64_t lq_buffer_elems(const lq_config *cfg, int32_t which);

/* Initialises `st` with configuration `cfg` and quantizes the FP32 state
 * S_init [B*H][d_v][d_k] (device, (16B)) into st->snap with the commit
 * quantizer ("LeapQuant: ...", Abstract and Figure 4: the largest outliers
 * become high-precision Compensator Tokens, the residual is smoothed across
 * channels and quantized once): compensator selection, residual smoothing,
 * per-row codes of lq_config.bits.  The residual's codes are taken with
 * exact FP32 quotients (R / c_j, then R' / sigma_i), so they are a function
 * of S_init alone.
 * With cfg.comp_rule = LQ_COMP_SVD the compensators are the r largest
 * singular triplets of each head's FP32 state, computed on the device by
 * subspace iteration: the Gram matrix S^T S, r + 8 basis vectors (at most
 * d_k; deterministic start vectors, or at a window commit the previous
 * compensators' k~_c in the first r), 16 iterations each orthonormalised by
 * an FP64 Cholesky factorisation, then a Rayleigh-Ritz step (FP64 Jacobi
 * eigensolver) on the basis.  Singular values and well-separated singular
 * vectors match an exact SVD to FP32 accuracy; vectors of nearly equal
 * singular values are a valid basis of their (ill-defined) subspace, not a
 * particular one.  It is much slower than LQ_COMP_ROWS (one CTA of 512
 * threads per head at init, prefill snapshots and every window commit).
 * S_init == NULL means the zero state.  Sets pos = 0 (also from
 * LQ_POS_PER_SEQUENCE). */
LQ_API lq_status lq_state_init(lq_state *st, const lq_config *cfg, const float *S_init,
                        lq_stream_t stream);

/* Decodes n_steps tokens (window positions pos+1 .. pos+n_steps) for every
 * sequence and head: for each token, u_t = v_t - S_{t-1} b_t and
 * o_t = S_t q_t computed from the fixed quantized boundary state plus the buffered
 * FP32 records ("LeapQuant: ...", Figure 2), and the record (L_t, k~_t, u_t)
 * is appended.  All n_steps tokens run inside one launch.
 * Requires 0 <= n_steps and pos + n_steps <= W (else LQ_ERR_WINDOW_FULL),
 * and pos != LQ_POS_PER_SEQUENCE (else LQ_ERR_WINDOW_OPEN);
 * n_steps == 0 is a no-op.  When cfg.auto_commit is set and the window
 * becomes full, the call also commits it (lq_window_commit, a second launch
 * on the same stream) and pos returns to 0; otherwise pos += n_steps.  If the
 * decode launch succeeded but the commit launch fails, the call returns
 * LQ_ERR_CUDA with the tokens decoded and pos == W (window full, not
 * committed); lq_window_commit completes it. */
LQ_API lq_status lq_decode_window(lq_state *st, const void *q, const void *k, const void *v,
                           const float *alpha, const float *beta, int32_t n_steps,
                           void *o, lq_stream_t stream);

/* Decode with per-sequence window positions (continuous batching): the
 * batch's sequences need not share a window position.  seq_pos (device,
 * int32 [B], 4-byte aligned, in/out) holds for each sequence b the number of
 * tokens buffered in its open window, 0 <= seq_pos[b] < W, or a negative
 * value for an idle slot.  One token per active sequence is decoded at window
 * position seq_pos[b] + 1 (q, k, v, alpha, beta, o laid out as for
 * lq_decode_window with n = 1; o of idle sequences is not written); every
 * sequence whose window becomes full is committed in the same call
 * (lq_window_commit's rule, on that sequence's heads only); then each active
 * seq_pos[b] advances to (seq_pos[b] + 1) mod W.  Three launches on `stream`
 * (decode, commit, position update).  Requires the batch-synchronous window
 * to be closed (pos == 0 or LQ_POS_PER_SEQUENCE, else LQ_ERR_WINDOW_OPEN) and
 * sets pos = LQ_POS_PER_SEQUENCE: windows may now be open on the device, so
 * the calls that need them closed refuse until lq_ragged_flush.  A position
 * >= W cannot be checked on the host: that sequence is skipped (its
 * position is left as it is) and the device error word records it
 * (LQ_DEVERR_BAD_POSITION).
 * If a later launch fails after an earlier one succeeded, LQ_ERR_CUDA is
 * returned with the earlier launches' effects in place. */
LQ_API lq_status lq_decode_ragged(lq_state *st, int32_t *seq_pos, const void *q, const void *k,
                           const void *v, const float *alpha, const float *beta, void *o,
                           lq_stream_t stream);

/* Window commit ("LeapQuant: ...", Figures 2 and 4): rebuilds the FP32
 * state S_pos = S^_0 D_{1..pos} + sum_m u_m (D_{m+1..pos} k~_m)^T, keeps its
 * r largest-norm rows as Compensator Tokens, smooths the residual across key
 * channels and re-quantizes it (codes of lq_config.bits) into st->snap; pos
 * returns to 0.
 * A no-op when pos == 0; LQ_ERR_WINDOW_OPEN when pos == LQ_POS_PER_SEQUENCE
 * (lq_ragged_flush commits per-sequence windows). */
LQ_API lq_status lq_window_commit(lq_state *st, lq_stream_t stream);

/* Closes every per-sequence window (the serving counterpart of
 * lq_window_commit; "LeapQuant: ...", Figure 2 and Figure 4, applied to each
 * sequence's own window): every sequence b with 1 <= seq_pos[b] < W commits
 * its seq_pos[b] buffered records exactly as lq_window_commit would, then
 * seq_pos[b] = 0.  Sequences at 0 or idle (negative) are untouched; a
 * position >= W is left as it is and reported (LQ_DEVERR_BAD_POSITION).
 * seq_pos: device int32 [B], 4-byte aligned, in/out (the array given to
 * lq_decode_ragged).  Requires pos == 0 or LQ_POS_PER_SEQUENCE (else
 * LQ_ERR_WINDOW_OPEN); sets pos = 0, after which snapshots, restores,
 * prefill and synchronous decode are allowed again.  W launches on `stream`
 * (one commit launch per buffered-record count 1 .. W-1 and the position
 * reset); if one fails, LQ_ERR_CUDA is returned with the earlier ones'
 * effects in place and pos unchanged. */
LQ_API lq_status lq_ragged_flush(lq_state *st, int32_t *seq_pos, lq_stream_t stream);

/* Prefill of T tokens from the FP32 state S_fp32 [B*H][d_v][d_k] (device,
 * (16B), in/out: the caller passes zeros for a fresh prompt; on return it
 * holds the state after the T tokens).  Outputs o [B, T, H, d_v].  After
 * every `snapshot_every` tokens the FP32 state is quantized (commit
 * quantizer) into snaps[i] (host array of T / snapshot_every snapshots
 * holding device pointers; may be NULL), one state per that many cached
 * tokens ("LeapQuant: ...", Figure 1(b)).  On return st->snap holds the
 * quantized state after T tokens, ready for decode.  The FP32 state is
 * carried across snapshots unquantized.
 *
 * workspace (device, (16B), workspace_bytes long; may be NULL with 0 bytes):
 * scratch of the chunked tensor-core prefill, used for the scalar gate with
 * BF16 io and d_k = 128.  Tokens are taken in chunks of 64 within each
 * snapshot interval, up to 16 chunks per pass of the workspace.  A
 * workspace of two full passes (lq_prefill_workspace_bytes) is used as two
 * halves: the next pass's chunk preparation runs while the current pass is
 * scanned; any smaller size of at least one chunk, 48 KB per sequence and
 * head, is used for one pass at a time of up to 16 chunks.
 * Without a usable workspace, for other shapes, and for the last
 * (snapshot_every mod 64) tokens of an interval, the recurrence runs token
 * by token on the FP32 state (same arithmetic, CUDA cores).  The caller
 * keeps the workspace alive until the call's work on `stream` has finished
 * and does not share it between concurrent calls.
 * The call runs its kernels on three internal streams of the current device
 * (the scans at the highest stream priority, the chunk preparation at the
 * lowest, snapshot quantization beside the next pass's preparation), forked
 * from `stream` by an event at the start and joined back into it at the end:
 * to the caller the work is ordered on `stream` like a single launch.  The
 * first call on each device creates those streams and events (held until the
 * process exits): make that first call before any stream capture.  Calls from
 * several host threads are serialized while they enqueue.
 * Requires pos == 0 (else LQ_ERR_WINDOW_OPEN; also LQ_POS_PER_SEQUENCE), T >= 0,
 * snapshot_every >= 1
 * and, when snaps != NULL, T % snapshot_every == 0.  T == 0 is a no-op. */
LQ_API lq_status lq_prefill_chunk(lq_state *st, float *S_fp32, const void *q, const void *k,
                           const void *v, const float *alpha, const float *beta,
                           int32_t T, int32_t snapshot_every, const lq_snapshot *snaps,
                           void *o, void *workspace, size_t workspace_bytes,
                           lq_stream_t stream);

/* lq_prefill_chunk for callers that cannot supply device memory of their
 * own -- for example a serving engine that reserved nearly all of HBM for its
 * pool at start-up and hands kernels only their input and output tensors, or
 * code that must not call cudaMalloc because it can synchronize the device.
 * The paper has no counterpart to this call; it exists for such callers.
 * Arguments and results are those of lq_prefill_chunk; the tensor-core
 * prefill's scratch comes from a fixed 8 MiB array inside the library (held
 * on every GPU that loads the library until the process exits) instead of a
 * workspace argument, and the call allocates nothing.
 *  - Limit: one chunk of scratch is 48 KB per sequence and head, so B * H
 *    may be at most 170 when the tensor-core path applies (scalar gate, BF16
 *    io, d_k = 128); above that the call returns LQ_ERR_UNSUPPORTED and does
 *    nothing.  Passes hold min(16, floor(170 / (B * H))) chunks.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and creates
 *    lq_prefill_chunk's internal streams and events (no device memory is
 *    allocated); make that first call before any stream capture.  A failed
 *    lookup returns LQ_ERR_CUDA.
 *  - All calls share the one array, which keeps the last call's contents
 *    (nothing in it needs to start at zero).  Calls whose work overlaps on
 *    the GPU (other streams, other host threads) race on it: serialize them. */
LQ_API lq_status lq_prefill_chunk_noalloc(lq_state *st, float *S_fp32, const void *q,
                                          const void *k, const void *v, const float *alpha,
                                          const float *beta, int32_t T, int32_t snapshot_every,
                                          const lq_snapshot *snaps, void *o, lq_stream_t stream);

/* Bytes of the workspace with which lq_prefill_chunk runs full passes of 16
 * chunks of 64 tokens, two passes in flight (2 x 16 x B x H x 48 KB); -1 for
 * an invalid configuration, 0 when the configuration has no tensor-core
 * prefill. */
LQ_API int64_t lq_prefill_workspace_bytes(const lq_config *cfg);

/* Copies the committed boundary state into `dst` (device buffers of the same
 * sizes): a prefix-cache snapshot, one quantized state kept per cached prefix
 * ("LeapQuant: ...", Figure 1(b): one state per 1,024 cached tokens).
 * Requires pos == 0 (else LQ_ERR_WINDOW_OPEN, also for LQ_POS_PER_SEQUENCE:
 * an open window's buffered tokens are not part of the snapshot). */
LQ_API lq_status lq_state_snapshot(const lq_state *st, const lq_snapshot *dst, lq_stream_t stream);

/* Copies a snapshot back into st->snap and sets pos = 0: resume from a
 * prefix-cache snapshot ("LeapQuant: ...", Figure 1(b)).  Requires pos == 0
 * (else LQ_ERR_WINDOW_OPEN, also for LQ_POS_PER_SEQUENCE). */
LQ_API lq_status lq_state_restore(lq_state *st, const lq_snapshot *src, lq_stream_t stream);

/* Comparator (not LeapQuant): n_steps of the recurrence on an FP32 state
 * S [B*H][d_v][d_k] (device, (16B), in/out) that is read and written every
 * step -- the FP32 per-step baseline of the paper's Table 2.  Uses cfg's
 * batch, heads, d_k, d_v, gate and io_dtype; inputs as lq_decode_window. */
LQ_API lq_status lq_fp32_step(const lq_config *cfg, float *S, const void *q, const void *k,
                       const void *v, const float *alpha, const float *beta,
                       int32_t n_steps, void *o, lq_stream_t stream);

/* Releases host resources of `st` (none today); device buffers stay the
 * caller's. */
LQ_API void lq_state_destroy(lq_state *st);

/* Static string naming a status. */
LQ_API const char *lq_status_string(lq_status s);

/* Bits of the device error word (lq_device_errors). */
#define LQ_DEVERR_WAIT_TIMEOUT 1u  /* a kernel gave up waiting for its own
                                      asynchronous copies (bounded wait
                                      expired); the affected outputs are not
                                      valid */
#define LQ_DEVERR_BAD_POSITION 2u  /* lq_decode_ragged / lq_ragged_flush met a
                                      per-sequence position >= W and skipped
                                      that sequence */

/* Reads and clears the library's device error word, an OR of LQ_DEVERR_*
 * bits (synchronizes the device). */
LQ_API lq_status lq_device_errors(uint32_t *flags);

#ifdef __cplusplus
}
#endif

#endif /* LQ_H */
