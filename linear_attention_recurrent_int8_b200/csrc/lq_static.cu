// lq_static.cu -- lq_prefill_chunk_noalloc: the prefill with its scratch in a
// fixed device array of this library instead of a caller-provided workspace.
//
// Some callers cannot hand the library extra device memory: a serving
// engine that reserved (almost) all of HBM for its own pool at start-up and
// gives kernels only the tensors they read and write; a plug-in that a host
// framework calls with input and output buffers and nothing else; code that
// must not call cudaMalloc because a cudaMalloc can synchronize the device
// and stall the other work on it.  For them this entry point takes the chunked
// prefill's scratch ([PT; T] of every chunk of a pass, 48 KB per chunk and
// head) from g_prefill_scratch below, a file-scope array of
// kStaticScratchBytes that every GPU which loads the library holds until the
// process exits.  It allocates nothing: no cudaMalloc, no cudaFree, no
// allocating library call.
//
// In host code the array's name refers to a host-side shadow, not to device
// memory: a kernel handed that name would fault, or on a system where the GPU
// can reach host memory would quietly work on the wrong bytes.  So the device
// address is looked up with cudaGetSymbolAddress the first time the entry
// point runs on a device (with that device current) and kept per device.
#include <cstdint>
#include <mutex>

#include "../../include/lq.h"
#include "lq_kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)8 << 20;  // 8 MiB

// Shared by every call on a device; it keeps whatever the last call wrote.
// Nothing in it has to start at zero: each pass writes every [PT; T] block
// it reads before reading it.
static __device__ __align__(256) unsigned char g_prefill_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices];  // device address of the array, per device (nullptr: not yet)

// The array's device address on the current device, looked up once per device.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_prefill_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

lq_status lq_prefill_chunk_noalloc(lq_state *st, float *S_fp32, const void *q, const void *k,
                                   const void *v, const float *alpha, const float *beta,
                                   int32_t T, int32_t snapshot_every, const lq_snapshot *snaps,
                                   void *o, lq_stream_t stream) {
    if (!st) return LQ_ERR_INVALID_ARGUMENT;
    // bytes of two 16-chunk passes (0: this shape has no chunked path, so no scratch)
    const int64_t two_passes = lq_prefill_workspace_bytes(&st->cfg);
    if (two_passes < 0) return LQ_ERR_INVALID_ARGUMENT;
    const int64_t one_chunk = two_passes / 32;
    if (one_chunk > (int64_t)kStaticScratchBytes) return LQ_ERR_UNSUPPORTED;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    if (one_chunk > 0 && T > 0) {
        if (scratch_address(&ws) != cudaSuccess) return LQ_ERR_CUDA;
        ws_bytes = kStaticScratchBytes;
    }
    return lq_prefill_chunk(st, S_fp32, q, k, v, alpha, beta, T, snapshot_every, snaps, o, ws,
                            ws_bytes, stream);
}

}  // extern "C"
