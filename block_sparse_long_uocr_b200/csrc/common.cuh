// common.cuh -- device helpers shared by the libuocr kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "uocr.h"

namespace uocr {

constexpr int kBlock = UOCR_BLOCK;        // tokens per KV block / page
constexpr int kLocal = UOCR_N_LOCAL;
constexpr int kRemote = UOCR_N_REMOTE;
constexpr int kSel = UOCR_N_SEL;
constexpr int kD = UOCR_HEAD_DIM;
constexpr int kDIdx = UOCR_IDX_DIM;
constexpr int kPageElems = kBlock * kD;   // elements of one (page, head) tile: 4096 bf16 = 8 KiB
constexpr float kLog2e = 1.4426950408889634f;
// Wall-time bound of every mbarrier wait in the library: far above any legitimate wait for an
// asynchronous copy or tensor-core operation (microseconds), short enough that a stuck wait
// ends the kernel with UOCR_DEVERR_TIMEOUT instead of hanging the device.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Query position and sequence for query i, with the device-side checks the
// ABI documents.  Returns false (and flags dev_err) when the query is invalid;
// p < 0 (empty sequence) is valid and means "no visible token".
struct QueryRef {
    int b;
    int p;
    int nb;
};

__device__ __forceinline__ void flag_error(int32_t *dev_err, uint32_t bits) {
    if (dev_err) atomicOr(reinterpret_cast<unsigned int *>(dev_err), bits);
}

// fixed_seq >= 0 puts every query in that sequence (a prefill chunk); otherwise
// query i belongs to q_seq[i], or to sequence i when q_seq is NULL.
__device__ __forceinline__ bool resolve_query(int i, const int32_t *seq_lens, const int32_t *q_seq,
                                              const int32_t *q_pos, int B, int max_blocks,
                                              int32_t *dev_err, bool report, QueryRef &r,
                                              int fixed_seq = -1) {
    int b = fixed_seq >= 0 ? fixed_seq : (q_seq ? __ldg(q_seq + i) : i);
    if (b < 0 || b >= B) {
        if (report) flag_error(dev_err, UOCR_DEVERR_POS);
        return false;
    }
    int len = __ldg(seq_lens + b);
    int p = q_pos ? __ldg(q_pos + i) : len - 1;
    if (p >= len || len > max_blocks * kBlock) {
        if (report) flag_error(dev_err, UOCR_DEVERR_POS);
        return false;
    }
    r.b = b;
    r.p = p;
    r.nb = p < 0 ? 0 : p / kBlock + 1;
    return true;
}

// 8 bf16 packed in a uint4 -> 8 floats (exact: bf16 is the top half of fp32).
__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f[2 * k] = __uint_as_float(w[k] << 16);
        f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
}

// A read-only load issued where it stands in the program: the volatile asm keeps the compiler
// from sinking a load issued ahead of a wait down to its first use after the wait.
__device__ __forceinline__ int ld_pinned(const int32_t *p) {
    int v;
    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Streaming 16-byte load that bypasses L1 allocation (each byte is read once).
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Transposed reduction of 16 partial sums over the 16 lanes of a half-warp.
// On entry lane l holds v[0..15], partial over its own slice of the reduced
// dimension; on exit v[0] of lane l is the full sum of index (l & 15).
// 8 + 4 + 2 + 1 = 15 shuffles instead of 16 x 4.
__device__ __forceinline__ float half_warp_transpose_sum16(float (&v)[16], int lane) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool hi = lane & 8;
        float send = hi ? v[k] : v[k + 8];
        float keep = hi ? v[k + 8] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const bool hi = lane & 4;
        float send = hi ? v[k] : v[k + 4];
        float keep = hi ? v[k + 4] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const bool hi = lane & 2;
        float send = hi ? v[k] : v[k + 2];
        float keep = hi ? v[k + 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    {
        const bool hi = lane & 1;
        float send = hi ? v[0] : v[1];
        float keep = hi ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
    return v[0];
}

// ---- shared-memory mbarrier + 1-D bulk copy (TMA) helpers
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy before a bulk copy signals it.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival on `bar` by the calling thread.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Global -> shared bulk copy completing `bytes` of transaction count on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// As mbar_try_wait, but the thread may be suspended for up to `hint_ns` while the phase is
// incomplete instead of returning at once (no spinning on the issue slots).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait on phase `parity` of `bar` for at most `timeout_ns` of wall time, giving up early
// when *abort becomes non-zero.  Returns true when the phase completed.  Each probe may
// suspend the thread for up to 20 us, so the wait does not spin.  A zero limit gives up at
// once without probing (the way the timeout paths are exercised).
__device__ __forceinline__ bool mbar_wait_timed(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                                const volatile int *abort) {
    if (timeout_ns == 0) return false;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (abort && *abort) return false;
        if (global_timer_ns() - t0 > timeout_ns) return false;
        if (it > (1u << 28)) return false;   // in case the timer does not advance
    }
}

// A drain wait (the copies or MMAs a warp issued must complete before its CTA ends or frees
// what they use): bounded like every wait, and a wait that runs out is reported as a timeout.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity, int32_t *dev_err) {
    if (!mbar_wait_timed(bar, parity, kWaitLimitNs, nullptr)) flag_error(dev_err, UOCR_DEVERR_TIMEOUT);
}

// Programmatic dependent launch: wait for the preceding grid's memory, and
// allow the next grid to begin launching.  Both are no-ops when the kernel was
// launched without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace uocr
