// lq_api.cu -- the C ABI of liblq (declared in include/lq.h): argument
// validation, status codes and kernel dispatch.  Every entry point validates
// all of its arguments before it launches anything, so a call that returns an
// error has no side effect.  No exception crosses the ABI.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/lq.h"
#include "lq_kernels.h"

namespace {

constexpr int kChunkTokens = 64;  // tokens per chunk of the tensor-core prefill
constexpr int kPassChunks = 16;   // chunks per pass of its workspace

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

lq_status check_config(const lq_config *c) {
    if (!c) return LQ_ERR_INVALID_ARGUMENT;
    if (c->batch < 1 || c->heads < 1) return LQ_ERR_INVALID_ARGUMENT;
    // B * H bounded so that every grid (at most 16 CTAs per head) and every
    // per-head int index stays far inside 2^31
    if ((int64_t)c->batch * c->heads > (1LL << 24)) return LQ_ERR_INVALID_ARGUMENT;
    if (c->d_k < 1 || c->d_v < 1) return LQ_ERR_INVALID_ARGUMENT;
    if ((c->d_k != 64 && c->d_k != 128) || (c->d_v != 64 && c->d_v != 128))
        return LQ_ERR_UNSUPPORTED;
    if (c->window < 1 || c->window > 32) return LQ_ERR_INVALID_ARGUMENT;
    if (c->n_comp < 0 || c->n_comp > 16 || c->n_comp > c->d_v) return LQ_ERR_INVALID_ARGUMENT;
    if (c->gate != LQ_GATE_SCALAR && c->gate != LQ_GATE_DIAG) return LQ_ERR_INVALID_ARGUMENT;
    if (c->io_dtype != LQ_F32 && c->io_dtype != LQ_BF16) return LQ_ERR_INVALID_ARGUMENT;
    if ((c->smoothing != 0 && c->smoothing != 1) || (c->auto_commit != 0 && c->auto_commit != 1) ||
        (c->delta != 0 && c->delta != 1))
        return LQ_ERR_INVALID_ARGUMENT;
    if (c->bits != 0 && c->bits != 8 && c->bits != 6 && c->bits != 4 && c->bits != 16)
        return LQ_ERR_INVALID_ARGUMENT;
    if (c->comp_rule != LQ_COMP_ROWS && c->comp_rule != LQ_COMP_SVD) return LQ_ERR_INVALID_ARGUMENT;
    if (c->comp_rule == LQ_COMP_SVD && c->n_comp > c->d_k) return LQ_ERR_INVALID_ARGUMENT;
    return LQ_OK;
}

// The SVD compensator rule is in effect (with r = 0 both rules are the same).
bool svd_rule(const lq_config *c) { return c->comp_rule == LQ_COMP_SVD && c->n_comp > 0; }

// Code width of a valid configuration (0 means 8).
int code_bits(const lq_config *c) { return c->bits == 0 ? 8 : c->bits; }

// Bytes of one head's residual: one per code, two codes per byte at 4 bits,
// two bytes per BF16 value at 16.
size_t code_bytes_per_head(const lq_config *c) {
    return (size_t)c->d_v * lq::code_row_bytes(lq::code_format(code_bits(c)), c->d_k);
}

// Elements of one head's residual in its storage type (int8, uint8 or bf16).
int64_t code_elems_per_head(const lq_config *c) {
    const int b = code_bits(c);
    return (int64_t)c->d_v * (b == 4 ? c->d_k / 2 : c->d_k);
}

lq_status check_snapshot(const lq_config *c, const lq_snapshot *s) {
    if (!s || !s->codes || !s->row_scale || !s->col_smooth) return LQ_ERR_INVALID_ARGUMENT;
    if (c->n_comp > 0 && (!s->comp_row || !s->comp_val)) return LQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(s->codes) || !aligned16(s->row_scale) || !aligned16(s->col_smooth))
        return LQ_ERR_MISALIGNED;
    if (c->n_comp > 0 && (!aligned16(s->comp_val) || !aligned_to(s->comp_row, 4)))
        return LQ_ERR_MISALIGNED;
    if (svd_rule(c) && !s->comp_u) return LQ_ERR_INVALID_ARGUMENT;
    if (svd_rule(c) && !aligned16(s->comp_u)) return LQ_ERR_MISALIGNED;
    return LQ_OK;
}

lq_status check_state(const lq_state *st) {
    if (!st) return LQ_ERR_INVALID_ARGUMENT;
    lq_status e = check_config(&st->cfg);
    if (e != LQ_OK) return e;
    e = check_snapshot(&st->cfg, &st->snap);
    if (e != LQ_OK) return e;
    if (!st->buf_gate || !st->buf_k || !st->buf_u) return LQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(st->buf_gate) || !aligned16(st->buf_k) || !aligned16(st->buf_u))
        return LQ_ERR_MISALIGNED;
    if ((st->pos < 0 && st->pos != LQ_POS_PER_SEQUENCE) || st->pos > st->cfg.window)
        return LQ_ERR_INVALID_ARGUMENT;
    return LQ_OK;
}

lq_status check_tokens(const lq_config *c, const void *q, const void *k, const void *v,
                       const float *alpha, const float *beta, const void *o) {
    if (!q || !k || !v || !alpha || !beta || !o) return LQ_ERR_INVALID_ARGUMENT;
    // q, k, v rows (and a diagonal gate's alpha rows) are moved with 16-byte
    // bulk copies and vector loads; o is written element by element
    const size_t es = c->io_dtype == LQ_BF16 ? 2 : 4;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned_to(o, es) ||
        !aligned_to(alpha, c->gate == LQ_GATE_DIAG ? 16 : 4) || !aligned_to(beta, 4))
        return LQ_ERR_MISALIGNED;
    return LQ_OK;
}

lq::DecodeArgs decode_args(const lq_state *st) {
    lq::DecodeArgs a{};
    a.codes = st->snap.codes;
    a.row_scale = st->snap.row_scale;
    a.col_smooth = st->snap.col_smooth;
    a.comp_row = st->cfg.n_comp > 0 ? st->snap.comp_row : nullptr;
    a.comp_val = st->cfg.n_comp > 0 ? st->snap.comp_val : nullptr;
    a.comp_u = svd_rule(&st->cfg) ? st->snap.comp_u : nullptr;
    a.buf_gate = st->buf_gate;
    a.buf_k = st->buf_k;
    a.buf_u = st->buf_u;
    a.B = st->cfg.batch;
    a.H = st->cfg.heads;
    a.W = st->cfg.window;
    a.delta = st->cfg.delta;
    a.R = st->cfg.n_comp;
    a.pos = st->pos;
    a.smoothing = st->cfg.smoothing;
    a.bits = code_bits(&st->cfg);
    return a;
}

lq::QuantArgs quant_args(const lq_config *c, const float *S, const lq_snapshot *s) {
    lq::QuantArgs a{};
    a.S = S;
    a.codes = s->codes;
    a.row_scale = s->row_scale;
    a.col_smooth = s->col_smooth;
    a.comp_row = c->n_comp > 0 ? s->comp_row : nullptr;
    a.comp_val = c->n_comp > 0 ? s->comp_val : nullptr;
    a.comp_u = svd_rule(c) ? s->comp_u : nullptr;
    a.BH = c->batch * c->heads;
    a.R = c->n_comp;
    a.smoothing = c->smoothing;
    a.bits = code_bits(c);
    return a;
}

lq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LQ_OK : LQ_ERR_CUDA; }

// Internal streams and events of the prefill, one set per device, created on
// first use and kept until the process exits.  The scans (the sequential
// chain) run on `chain` at the highest stream priority; the chunk preparation
// of the next pass runs on `prep` at the lowest, into the other half of a
// double workspace, on the SMs the scan leaves free; snapshot quantization
// runs on `snap` while the next pass is prepared.  Each call forks them from
// the caller's stream and joins them back, so the call keeps stream order
// (and works inside a stream capture once the set exists).
struct PrefillStreams {
    cudaStream_t chain, prep, snap;
    cudaEvent_t fork, join, prep_done[2], scan_done[2], snap_in, snap_done;
};

std::mutex g_prefill_mutex;  // guards the sets and each call's enqueue sequence

// The current device's set (nullptr for device ordinals past 63, which then
// run everything on the caller's stream).  Called with g_prefill_mutex held.
cudaError_t prefill_streams(PrefillStreams **out) {
    static PrefillStreams sets[64];
    static bool ready[64];
    *out = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaSuccess;
    PrefillStreams &p = sets[dev];
    if (!ready[dev]) {
        int least = 0, greatest = 0;
        e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        cudaStream_t *streams[3] = {&p.chain, &p.prep, &p.snap};
        const int prio[3] = {greatest, least, greatest};
        cudaEvent_t *events[8] = {&p.fork, &p.join, &p.prep_done[0], &p.prep_done[1],
                                  &p.scan_done[0], &p.scan_done[1], &p.snap_in, &p.snap_done};
        int ns = 0, nev = 0;  // created so far
        while (e == cudaSuccess && ns < 3) {
            e = cudaStreamCreateWithPriority(streams[ns], cudaStreamNonBlocking, prio[ns]);
            if (e == cudaSuccess) ++ns;
        }
        while (e == cudaSuccess && nev < 8) {
            e = cudaEventCreateWithFlags(events[nev], cudaEventDisableTiming);
            if (e == cudaSuccess) ++nev;
        }
        if (e != cudaSuccess) {
            for (int i = 0; i < nev; ++i) cudaEventDestroy(*events[i]);
            for (int i = 0; i < ns; ++i) cudaStreamDestroy(*streams[i]);
            return e;
        }
        ready[dev] = true;
    }
    *out = &p;
    return cudaSuccess;
}

lq_status copy_snapshot(const lq_config *c, const lq_snapshot *dst, const lq_snapshot *src,
                        cudaStream_t stream) {
    const size_t bh = (size_t)c->batch * c->heads;
    const cudaMemcpyKind kind = cudaMemcpyDeviceToDevice;
    cudaError_t e = cudaMemcpyAsync(dst->codes, src->codes, bh * code_bytes_per_head(c), kind, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dst->row_scale, src->row_scale, bh * c->d_v * 4, kind, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dst->col_smooth, src->col_smooth, bh * c->d_k * 4, kind, stream);
    if (e == cudaSuccess && c->n_comp > 0)
        e = cudaMemcpyAsync(dst->comp_row, src->comp_row, bh * c->n_comp * 4, kind, stream);
    if (e == cudaSuccess && c->n_comp > 0)
        e = cudaMemcpyAsync(dst->comp_val, src->comp_val, bh * c->n_comp * c->d_k * 4, kind,
                            stream);
    if (e == cudaSuccess && svd_rule(c))
        e = cudaMemcpyAsync(dst->comp_u, src->comp_u, bh * c->n_comp * c->d_v * 4, kind, stream);
    return cuda_status(e);
}

}  // namespace

extern "C" {

int64_t lq_buffer_elems(const lq_config *cfg, int32_t which) {
    if (check_config(cfg) != LQ_OK) return -1;
    const int64_t bh = (int64_t)cfg->batch * cfg->heads;
    const int64_t G = cfg->gate == LQ_GATE_DIAG ? cfg->d_k : 1;
    switch (which) {
        case 0: return bh * code_elems_per_head(cfg);
        case 1: return bh * cfg->d_v;
        case 2: return bh * cfg->d_k;
        case 3: return bh * cfg->n_comp;
        case 4: return bh * cfg->n_comp * cfg->d_k;
        case 5: return bh * cfg->window * G;
        case 6: return bh * cfg->window * cfg->d_k;
        case 7: return bh * cfg->window * cfg->d_v;
        case 8: return cfg->comp_rule == LQ_COMP_SVD ? bh * cfg->n_comp * cfg->d_v : 0;
        default: return -1;
    }
}

lq_status lq_state_init(lq_state *st, const lq_config *cfg, const float *S_init,
                        lq_stream_t stream) {
    if (!st) return LQ_ERR_INVALID_ARGUMENT;
    lq_status e = check_config(cfg);
    if (e != LQ_OK) return e;
    lq_state tmp = *st;
    tmp.cfg = *cfg;
    tmp.pos = 0;
    e = check_state(&tmp);
    if (e != LQ_OK) return e;
    if (S_init && !aligned16(S_init)) return LQ_ERR_MISALIGNED;
    e = cuda_status(lq::launch_quantize(quant_args(cfg, S_init, &tmp.snap), cfg->d_k, cfg->d_v,
                                        (cudaStream_t)stream));
    if (e != LQ_OK) return e;
    st->cfg = *cfg;
    st->pos = 0;
    st->impl = nullptr;
    return LQ_OK;
}

lq_status lq_decode_window(lq_state *st, const void *q, const void *k, const void *v,
                           const float *alpha, const float *beta, int32_t n_steps, void *o,
                           lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos == LQ_POS_PER_SEQUENCE) return LQ_ERR_WINDOW_OPEN;
    if (n_steps < 0) return LQ_ERR_INVALID_ARGUMENT;
    if (n_steps == 0) return LQ_OK;
    if (st->pos + n_steps > st->cfg.window) return LQ_ERR_WINDOW_FULL;
    e = check_tokens(&st->cfg, q, k, v, alpha, beta, o);
    if (e != LQ_OK) return e;
    lq::DecodeArgs a = decode_args(st);
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.o = o;
    a.n_steps = n_steps;
    e = cuda_status(lq::launch_decode(a, st->cfg.d_k, st->cfg.d_v, st->cfg.gate,
                                      st->cfg.io_dtype == LQ_BF16, (cudaStream_t)stream));
    if (e != LQ_OK) return e;
    st->pos += n_steps;
    if (st->cfg.auto_commit && st->pos == st->cfg.window) return lq_window_commit(st, stream);
    return LQ_OK;
}

lq_status lq_decode_ragged(lq_state *st, int32_t *seq_pos, const void *q, const void *k,
                           const void *v, const float *alpha, const float *beta, void *o,
                           lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos != 0 && st->pos != LQ_POS_PER_SEQUENCE) return LQ_ERR_WINDOW_OPEN;
    if (!seq_pos) return LQ_ERR_INVALID_ARGUMENT;
    if (!aligned_to(seq_pos, 4)) return LQ_ERR_MISALIGNED;
    e = check_tokens(&st->cfg, q, k, v, alpha, beta, o);
    if (e != LQ_OK) return e;
    const int W = st->cfg.window;
    lq::DecodeArgs a = decode_args(st);
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.o = o;
    a.seq_pos = seq_pos;
    // one token per active sequence; stages laid out for W - 1 buffered records
    a.pos = W - 1;
    a.n_steps = 1;
    cudaStream_t s = (cudaStream_t)stream;
    e = cuda_status(lq::launch_decode(a, st->cfg.d_k, st->cfg.d_v, st->cfg.gate,
                                      st->cfg.io_dtype == LQ_BF16, s));
    if (e != LQ_OK) return e;
    // from here on windows may be open on the device
    st->pos = LQ_POS_PER_SEQUENCE;
    // the sequences whose window is now full (seq_pos == W - 1) commit W records
    a.pos = W;
    a.n_steps = 0;
    a.commit_match = W - 1;
    e = cuda_status(lq::launch_commit(a, st->cfg.d_k, st->cfg.d_v, st->cfg.gate, s));
    if (e != LQ_OK) return e;
    return cuda_status(lq::launch_advance_positions(seq_pos, st->cfg.batch, W, s));
}

lq_status lq_ragged_flush(lq_state *st, int32_t *seq_pos, lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos != 0 && st->pos != LQ_POS_PER_SEQUENCE) return LQ_ERR_WINDOW_OPEN;
    if (!seq_pos) return LQ_ERR_INVALID_ARGUMENT;
    if (!aligned_to(seq_pos, 4)) return LQ_ERR_MISALIGNED;
    const int W = st->cfg.window;
    cudaStream_t s = (cudaStream_t)stream;
    lq::DecodeArgs a = decode_args(st);
    a.seq_pos = seq_pos;
    a.n_steps = 0;
    // one commit launch per record count p: the sequences holding p records
    for (int p = 1; p < W; ++p) {
        a.pos = p;
        a.commit_match = p;
        e = cuda_status(lq::launch_commit(a, st->cfg.d_k, st->cfg.d_v, st->cfg.gate, s));
        if (e != LQ_OK) return e;
    }
    e = cuda_status(lq::launch_reset_positions(seq_pos, st->cfg.batch, W, s));
    if (e != LQ_OK) return e;
    st->pos = 0;
    return LQ_OK;
}

lq_status lq_window_commit(lq_state *st, lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos == LQ_POS_PER_SEQUENCE) return LQ_ERR_WINDOW_OPEN;
    if (st->pos == 0) return LQ_OK;
    lq::DecodeArgs a = decode_args(st);
    a.n_steps = 0;
    e = cuda_status(lq::launch_commit(a, st->cfg.d_k, st->cfg.d_v, st->cfg.gate, (cudaStream_t)stream));
    if (e != LQ_OK) return e;
    st->pos = 0;
    return LQ_OK;
}

int64_t lq_prefill_workspace_bytes(const lq_config *cfg) {
    if (check_config(cfg) != LQ_OK) return -1;
    if (!lq::chunk_path_supported(cfg->d_k, cfg->d_v, cfg->gate, cfg->io_dtype == LQ_BF16)) return 0;
    // two full passes: one prepared while the other is scanned
    return (int64_t)lq::chunk_workspace_bytes(cfg->batch * cfg->heads, 2 * kPassChunks);
}

lq_status lq_prefill_chunk(lq_state *st, float *S_fp32, const void *q, const void *k,
                           const void *v, const float *alpha, const float *beta, int32_t T,
                           int32_t snapshot_every, const lq_snapshot *snaps, void *o,
                           void *workspace, size_t workspace_bytes, lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos != 0) return LQ_ERR_WINDOW_OPEN;
    if (T < 0 || snapshot_every < 1) return LQ_ERR_INVALID_ARGUMENT;
    if (T == 0) return LQ_OK;
    if (snaps && T % snapshot_every != 0) return LQ_ERR_INVALID_ARGUMENT;
    if (!S_fp32) return LQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(S_fp32)) return LQ_ERR_MISALIGNED;
    if (!workspace != (workspace_bytes == 0)) return LQ_ERR_INVALID_ARGUMENT;
    if (workspace && !aligned16(workspace)) return LQ_ERR_MISALIGNED;
    e = check_tokens(&st->cfg, q, k, v, alpha, beta, o);
    if (e != LQ_OK) return e;
    if (snaps) {
        const int n = T / snapshot_every;
        for (int i = 0; i < n; ++i) {
            e = check_snapshot(&st->cfg, &snaps[i]);
            if (e != LQ_OK) return e;
        }
    }
    const lq_config *c = &st->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    lq::RecurArgs r{};
    r.S = S_fp32;
    r.q = q;
    r.k = k;
    r.v = v;
    r.alpha = alpha;
    r.beta = beta;
    r.o = o;
    r.B = c->batch;
    r.delta = c->delta;
    r.H = c->heads;
    r.T_total = T;
    lq::ChunkArgs ca{};
    ca.S = S_fp32;
    ca.alpha = alpha;
    ca.beta = beta;
    ca.o = o;
    ca.B = c->batch;
    ca.H = c->heads;
    ca.DV = c->d_v;
    ca.T_total = T;
    ca.delta = c->delta;

    std::lock_guard<std::mutex> lock(g_prefill_mutex);
    PrefillStreams *ps = nullptr;
    e = cuda_status(prefill_streams(&ps));
    if (e != LQ_OK) return e;
    // chunks per pass of the tensor-core path (0: token by token); two
    // workspace halves (the next pass prepared while this one is scanned)
    // when the workspace holds two full passes
    const int BH = c->batch * c->heads;
    int pass = 0, nbuf = 1;
    size_t per = 0;
    if (workspace && lq::chunk_path_supported(c->d_k, c->d_v, c->gate, c->io_dtype == LQ_BF16)) {
        per = lq::chunk_workspace_bytes(BH, 1);
        const size_t chunks = workspace_bytes / per;
        if (ps && chunks >= 2 * (size_t)kPassChunks) nbuf = 2;
        pass = (int)(chunks < (size_t)kPassChunks ? chunks : kPassChunks);
    }
    cudaStream_t chain = s, prep = s, snap = s;
    cudaError_t ce = cudaSuccess;
    if (ps) {
        chain = ps->chain;
        prep = nbuf == 2 ? ps->prep : ps->chain;
        snap = ps->snap;
        ce = cudaEventRecord(ps->fork, s);
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(ps->chain, ps->fork, 0);
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(ps->prep, ps->fork, 0);
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(ps->snap, ps->fork, 0);
        if (ce != cudaSuccess) return cuda_status(ce);
    }
    // a snapshot quantization on `snap` reads the state: the chain waits for
    // it before it writes the state again
    bool snap_pending = false;
    auto wait_snap = [&]() -> cudaError_t {
        if (!snap_pending) return cudaSuccess;
        snap_pending = false;
        return cudaStreamWaitEvent(chain, ps->snap_done, 0);
    };
    unsigned char *wsb = static_cast<unsigned char *>(workspace);
    int g = 0;  // passes so far
    for (int t0 = 0, i = 0; ce == cudaSuccess && t0 < T; t0 += snapshot_every, ++i) {
        const int nt = T - t0 < snapshot_every ? T - t0 : snapshot_every;
        int done = 0;
        if (pass > 0) {
            // whole chunks of this interval on the tensor cores, in passes
            const int nch = nt / kChunkTokens;
            for (int c0 = 0; ce == cudaSuccess && c0 < nch; c0 += pass, ++g) {
                const int buf = g % nbuf;
                ca.t0 = t0 + c0 * kChunkTokens;
                ca.nc = nch - c0 < pass ? nch - c0 : pass;
                ca.ws = reinterpret_cast<float *>(wsb + (size_t)buf * pass * per);
                if (nbuf == 2) {
                    // the half's previous reader, the scan of pass g - 2, is done
                    if (g >= 2) ce = cudaStreamWaitEvent(prep, ps->scan_done[buf], 0);
                    if (ce == cudaSuccess) ce = lq::launch_chunk_prep(ca, q, k, prep);
                    if (ce == cudaSuccess) ce = cudaEventRecord(ps->prep_done[buf], prep);
                    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(chain, ps->prep_done[buf], 0);
                } else {
                    ce = lq::launch_chunk_prep(ca, q, k, chain);
                }
                if (ce == cudaSuccess) ce = wait_snap();
                if (ce == cudaSuccess) ce = lq::launch_chunk_scan(ca, q, k, v, chain);
                if (ce == cudaSuccess && nbuf == 2) ce = cudaEventRecord(ps->scan_done[buf], chain);
            }
            done = nch * kChunkTokens;
        }
        if (ce == cudaSuccess && done < nt) {
            r.t0 = t0 + done;
            r.nt = nt - done;
            ce = wait_snap();
            if (ce == cudaSuccess)
                ce = lq::launch_recurrence(r, c->d_k, c->d_v, c->gate, c->io_dtype == LQ_BF16, true, chain);
        }
        if (ce == cudaSuccess && snaps) {
            if (ps) {
                ce = cudaEventRecord(ps->snap_in, chain);
                if (ce == cudaSuccess) ce = cudaStreamWaitEvent(snap, ps->snap_in, 0);
                if (ce == cudaSuccess)
                    ce = lq::launch_quantize(quant_args(c, S_fp32, &snaps[i]), c->d_k, c->d_v, snap);
                if (ce == cudaSuccess) ce = cudaEventRecord(ps->snap_done, snap);
                snap_pending = ce == cudaSuccess;
            } else {
                ce = lq::launch_quantize(quant_args(c, S_fp32, &snaps[i]), c->d_k, c->d_v, chain);
            }
        }
    }
    if (ce == cudaSuccess) ce = wait_snap();
    if (ce == cudaSuccess) ce = lq::launch_quantize(quant_args(c, S_fp32, &st->snap), c->d_k, c->d_v, chain);
    if (ps) {
        // join every internal stream back into the caller's stream (also
        // after a failed launch, so that later work on it stays ordered)
        for (cudaStream_t x : {ps->prep, ps->snap, ps->chain}) {
            cudaError_t je = cudaEventRecord(ps->join, x);
            if (je == cudaSuccess) je = cudaStreamWaitEvent(s, ps->join, 0);
            if (ce == cudaSuccess) ce = je;
        }
    }
    return cuda_status(ce);
}

lq_status lq_state_snapshot(const lq_state *st, const lq_snapshot *dst, lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos != 0) return LQ_ERR_WINDOW_OPEN;
    e = check_snapshot(&st->cfg, dst);
    if (e != LQ_OK) return e;
    return copy_snapshot(&st->cfg, dst, &st->snap, (cudaStream_t)stream);
}

lq_status lq_state_restore(lq_state *st, const lq_snapshot *src, lq_stream_t stream) {
    lq_status e = check_state(st);
    if (e != LQ_OK) return e;
    if (st->pos != 0) return LQ_ERR_WINDOW_OPEN;
    e = check_snapshot(&st->cfg, src);
    if (e != LQ_OK) return e;
    e = copy_snapshot(&st->cfg, &st->snap, src, (cudaStream_t)stream);
    if (e == LQ_OK) st->pos = 0;
    return e;
}

lq_status lq_fp32_step(const lq_config *cfg, float *S, const void *q, const void *k,
                       const void *v, const float *alpha, const float *beta, int32_t n_steps,
                       void *o, lq_stream_t stream) {
    lq_status e = check_config(cfg);
    if (e != LQ_OK) return e;
    if (n_steps < 0) return LQ_ERR_INVALID_ARGUMENT;
    if (n_steps == 0) return LQ_OK;
    if (!S) return LQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(S)) return LQ_ERR_MISALIGNED;
    e = check_tokens(cfg, q, k, v, alpha, beta, o);
    if (e != LQ_OK) return e;
    lq::RecurArgs r{};
    r.S = S;
    r.q = q;
    r.k = k;
    r.v = v;
    r.alpha = alpha;
    r.beta = beta;
    r.o = o;
    r.B = cfg->batch;
    r.delta = cfg->delta;
    r.H = cfg->heads;
    r.T_total = n_steps;
    r.t0 = 0;
    r.nt = n_steps;
    return cuda_status(lq::launch_recurrence(r, cfg->d_k, cfg->d_v, cfg->gate,
                                             cfg->io_dtype == LQ_BF16, false, (cudaStream_t)stream));
}

void lq_state_destroy(lq_state *st) {
    if (st) st->impl = nullptr;
}

const char *lq_status_string(lq_status s) {
    switch (s) {
        case LQ_OK: return "LQ_OK";
        case LQ_ERR_INVALID_ARGUMENT: return "LQ_ERR_INVALID_ARGUMENT";
        case LQ_ERR_UNSUPPORTED: return "LQ_ERR_UNSUPPORTED";
        case LQ_ERR_WINDOW_FULL: return "LQ_ERR_WINDOW_FULL";
        case LQ_ERR_WINDOW_OPEN: return "LQ_ERR_WINDOW_OPEN";
        case LQ_ERR_MISALIGNED: return "LQ_ERR_MISALIGNED";
        case LQ_ERR_CUDA: return "LQ_ERR_CUDA";
    }
    return "LQ_UNKNOWN_STATUS";
}

lq_status lq_device_errors(uint32_t *flags) {
    if (!flags) return LQ_ERR_INVALID_ARGUMENT;
    unsigned int v = 0;
    const cudaError_t e = lq::read_and_clear_dev_error(&v);
    *flags = v;
    return cuda_status(e);
}

}  // extern "C"
