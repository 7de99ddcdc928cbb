// lq_common.cuh -- device helpers shared by the liblq kernels (sm_100a).
//
// * 1-D bulk copies global -> shared (cp.async.bulk, the TMA's untiled form,
//   no multicast) completing on an mbarrier, and a bounded wait on it.
// * Warp reductions (butterfly and transposing), io conversions.
// * The library's device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lq {

// Device error word, read and cleared by lq_device_errors().
extern __device__ unsigned int g_dev_error;
constexpr unsigned int kErrWaitTimeout = 1u;
constexpr unsigned int kErrBadPosition = 2u;  // a per-sequence window position >= W

// A bounded wait gives up after this many nanoseconds of global time.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
    // make the initialised barrier visible to the async (TMA) proxy
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

// Bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing `bytes` transactions on bar.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bulk prefetch of `bytes` (multiple of 16, address 16-byte aligned) of
// global memory into L2.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// 4-byte asynchronous copy global -> shared (both 4-byte aligned).
__device__ __forceinline__ void cp_async4(void *dst_smem, const void *src_gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem)
                 : "memory");
}

// 16-byte global -> shared copy (both addresses 16-byte aligned), bypassing L1.
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src_gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem)
                 : "memory");
}

// Closes the group of this thread's cp.async copies issued so far; waits
// until all of its groups have completed.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Makes `bar` track completion of this thread's earlier cp.async copies: its
// pending arrival count is raised by one now and lowered when they complete.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tests phase `parity` of `bar`; while it is incomplete the thread may be
// suspended (not spinning) for up to kSuspendHintNs, and resumes as soon as
// the phase completes.
constexpr uint32_t kSuspendHintNs = 100000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, "
        "0, p; }"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendHintNs)
        : "memory");
    return done != 0;
}

// Waits for phase `parity` of `bar` to complete, for at most kWaitLimitNs.
// On expiry it records kErrWaitTimeout in the device error word and returns
// false; the caller then skips its work (its outputs are not valid).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        // the clock is read once every 16 tests
        for (int k = 0; k < 16; ++k)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_dev_error, kErrWaitTimeout);
            return false;
        }
    }
}

// Named barrier ID over NT threads (ID 0 is __syncthreads).
template <int ID, int NT>
__device__ __forceinline__ void named_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(NT) : "memory");
}

// Named barrier ID over NT threads that also ORs `pred` over them: every
// participant gets the same answer (so a group can leave a loop together).
template <int ID, int NT>
__device__ __forceinline__ bool named_sync_or(bool pred) {
    uint32_t out;
    asm volatile(
        "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, %2, %3, p; selp.u32 %0, 1, 0, "
        "q; }"
        : "=r"(out)
        : "r"((uint32_t)pred), "n"(ID), "n"(NT)
        : "memory");
    return out != 0;
}

// Named barrier 1 over the first NT threads of the CTA (the consumer warps of
// a warp-specialised kernel; barrier 0 is __syncthreads).
template <int NT>
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// Same barrier, returning whether `pred` was true in any participating thread.
template <int NT>
__device__ __forceinline__ bool consumer_sync_or(bool pred) {
    uint32_t out;
    asm volatile(
        "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, 1, %2, p; selp.u32 %0, 1, 0, "
        "q; }"
        : "=r"(out)
        : "r"((uint32_t)pred), "n"(NT)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar))
                 : "memory");
}

// Orders this thread's generic-proxy shared-memory accesses before later
// asynchronous-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Warp reductions
// ---------------------------------------------------------------------------

// Sum over aligned groups of WIDTH lanes (butterfly; every lane gets the sum).
template <int WIDTH>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int s = WIDTH / 2; s > 0; s >>= 1) x += __shfl_xor_sync(0xffffffffu, x, s);
    return x;
}

template <int WIDTH>
__device__ __forceinline__ float group_max(float x) {
#pragma unroll
    for (int s = WIDTH / 2; s > 0; s >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, s));
    return x;
}

// Transposing reduction: each lane holds N partial values; the N sums are
// taken over aligned groups of WIDTH lanes.  Each halving step exchanges half
// of the remaining values with the partner lane, so N values cost about N
// shuffles instead of N*log2(WIDTH).  On return v[0] holds the sum of value
// index transposed_index<N, WIDTH>(lane).
template <int N, int S>
__device__ __forceinline__ void transposed_sum_step(float *v, int lane) {
    if constexpr (S > 0) {
        if constexpr (N > 1) {
            const bool upper = (lane & S) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                float send = upper ? v[i] : v[i + N / 2];
                float keep = upper ? v[i + N / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, S);
            }
            transposed_sum_step<N / 2, S / 2>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], S);
            transposed_sum_step<1, S / 2>(v, lane);
        }
    }
}

template <int N, int WIDTH>
__device__ __forceinline__ void transposed_sum(float (&v)[N], int lane) {
    transposed_sum_step<N, WIDTH / 2>(v, lane);
}

// Same as transposed_sum with max instead of sum.
template <int N, int S>
__device__ __forceinline__ void transposed_max_step(float *v, int lane) {
    if constexpr (S > 0) {
        if constexpr (N > 1) {
            const bool upper = (lane & S) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                float send = upper ? v[i] : v[i + N / 2];
                float keep = upper ? v[i + N / 2] : v[i];
                v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, S));
            }
            transposed_max_step<N / 2, S / 2>(v, lane);
        } else {
            v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], S));
            transposed_max_step<1, S / 2>(v, lane);
        }
    }
}

template <int N, int WIDTH>
__device__ __forceinline__ void transposed_max(float (&v)[N], int lane) {
    transposed_max_step<N, WIDTH / 2>(v, lane);
}

// A lane offset (within its WIDTH-lane group) that holds value index n after
// a transposed reduction of N values.
template <int N, int S>
__host__ __device__ constexpr int transposed_owner_step(int n) {
    if constexpr (S > 0 && N > 1)
        return (n >= N / 2 ? S : 0) + transposed_owner_step<N / 2, S / 2>(n >= N / 2 ? n - N / 2 : n);
    else
        return 0;
}

template <int N, int WIDTH>
__host__ __device__ constexpr int transposed_owner(int n) {
    return transposed_owner_step<N, WIDTH / 2>(n);
}

template <int N, int S>
__device__ __forceinline__ int transposed_index_step(int lane) {
    if constexpr (S > 0 && N > 1)
        return ((lane & S) ? N / 2 : 0) + transposed_index_step<N / 2, S / 2>(lane);
    else
        return 0;
}

template <int N, int WIDTH>
__device__ __forceinline__ int transposed_index(int lane) {
    return transposed_index_step<N, WIDTH / 2>(lane);
}

// ---------------------------------------------------------------------------
// int8 codes -> FP32, io conversions
// ---------------------------------------------------------------------------

// Exact int -> FP32 for |a| < 2^22 on the integer/FP32 pipes: the bits of
// 1.5 * 2^23 + a, minus 1.5 * 2^23.
__device__ __forceinline__ float small_int_to_f32(int a) {
    return __int_as_float(0x4B400000 + a) - 12582912.0f;
}

// Four int8 codes packed in a 32-bit word -> four exact FP32 values.  Each
// biased byte (Q + 128) is placed in the low mantissa bits of 2^23, giving
// 2^23 + Q + 128 exactly; one subtraction recovers Q.
__device__ __forceinline__ void codes4_to_f32(uint32_t w, float (&f)[4]) {
    const uint32_t u = w ^ 0x80808080u;
    f[0] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)) - 8388736.0f;
    f[1] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)) - 8388736.0f;
    f[2] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)) - 8388736.0f;
    f[3] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653)) - 8388736.0f;
}

// N consecutive floats (N = 2 or 4, address 8- or 16-byte aligned).
template <int N>
__device__ __forceinline__ void load_vec(float (&v)[N], const float *p) {
    if constexpr (N == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        v[0] = x.x, v[1] = x.y, v[2] = x.z, v[3] = x.w;
    } else {
        static_assert(N == 2, "vector width");
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x, v[1] = x.y;
    }
}

template <int N>
__device__ __forceinline__ void store_vec(float *p, const float (&v)[N]) {
    if constexpr (N == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
        static_assert(N == 2, "vector width");
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    }
}

template <bool BF16>
__device__ __forceinline__ float load_io(const void *p, size_t i) {
    if constexpr (BF16)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    else
        return static_cast<const float *>(p)[i];
}

// N consecutive io elements starting at element i (N = 2 or 4; element
// address aligned to N elements).
template <bool BF16, int N>
__device__ __forceinline__ void load_io_vec(float (&v)[N], const void *p, size_t i) {
    if constexpr (BF16) {
        const __nv_bfloat162 *q = reinterpret_cast<const __nv_bfloat162 *>(
            static_cast<const __nv_bfloat16 *>(p) + i);
#pragma unroll
        for (int e = 0; e < N / 2; ++e) {
            const float2 f = __bfloat1622float2(q[e]);
            v[2 * e] = f.x, v[2 * e + 1] = f.y;
        }
    } else {
        load_vec<N>(v, static_cast<const float *>(p) + i);
    }
}

template <bool BF16>
__device__ __forceinline__ void store_io(void *p, size_t i, float x) {
    if constexpr (BF16)
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
    else
        static_cast<float *>(p)[i] = x;
}

}  // namespace lq
