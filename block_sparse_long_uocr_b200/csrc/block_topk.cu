// block_topk.cu -- per-query block selection: 4 local blocks + top-12 remote.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 step 3:
// each query keeps 16 blocks, the 4 most recent ("local", the 128-token
// window) and the 12 remote blocks with the highest indexer score; inference
// uses a hard top-k.  Ranking: score descending, then lower block id.
//
// One CTA of 512 threads per query; every candidate's ranking key is the
// 64-bit composite (order-preserving fp32 key << 32 | ~id): distinct, larger
// for a higher score and, among equal scores, for the lower id.
//   1. The candidates' scores are read once from L2 (the scan just wrote them)
//      into shared memory as order-preserving keys.
//   2. Threshold: the 12th largest of the 16 warp maxima.  Those 12 maxima are
//      12 distinct candidates at or above it, so every member of the top 12 is
//      at or above it too.
//   3. Survivors (keys >= threshold; typically a few dozen) are appended to a
//      shared list; each survivor's rank is the number of survivors with a
//      larger composite, and ranks 0..11 are the answer.
//   4. One warp writes the 12 ids in ascending order plus the 4 local blocks.
// If the survivors overflow their list (heavily tied scores) the CTA falls
// back to an exact two-level extraction: every warp takes its top 12 by 12
// rounds of a warp-wide max, then one warp takes the top 12 of those.
// Rows longer than the shared-memory budget are read from L2 instead of staged.
// An optional per-sequence candidate bitmap (the walk-through's page-aware
// candidate constraint, section 五 image_bucket_constraint) excludes remote
// candidates before the ranking; the local window is always kept.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSmemKeys = 48 * 1024;    // stage rows up to 48K candidates (192 KiB of keys)
constexpr int kSurvivorCap = 2048;          // survivor list capacity (16 KiB)

// Larger key <=> larger float; -0 and +0 map to the same key (they compare equal).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = (f == 0.0f) ? 0u : __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t composite(uint32_t key, int j) {
    return ((uint64_t)key << 32) | (uint32_t)(~(uint32_t)j);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

// Keys of one query's candidates: staged in shared memory, or read from the scores row.
// A candidate that the optional candidate mask excludes gets key 0, below every real key
// (order_key never returns 0 for a non-NaN score).
struct KeySource {
    const uint32_t *smem;
    const float *row;
    const uint32_t *mask;   // this sequence's candidate bitmap, or NULL
    __device__ __forceinline__ uint32_t raw(int j) const {
        if (mask && !((__ldg(mask + (j >> 5)) >> (j & 31)) & 1u)) return 0u;
        return order_key(__ldcg(row + j));
    }
    __device__ __forceinline__ uint32_t operator()(int j) const { return smem ? smem[j] : raw(j); }
};

// Largest composite strictly below `cap` among candidates j = first, first + stride, ... < n
// (0 when there is none; a real composite is never 0 because ~j != 0 for j < 2^31 - 1).
__device__ __forceinline__ uint64_t best_below(const KeySource &key, int first, int stride, int n,
                                               uint64_t cap) {
    uint64_t best = 0;
    for (int j = first; j < n; j += stride) {
        const uint64_t c = composite(key(j), j);
        if (c < cap && c > best) best = c;
    }
    return best;
}

// Exact fallback: the top kRemote composites of candidates [0, nc) into out_c[0..11].
// Called by every thread of the CTA.
__device__ void topk_two_level(const KeySource &key, int nc, uint64_t *s_cand, uint64_t *out_c) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t cap = ~0ull;
    uint64_t mine = best_below(key, tid, kTopkThreads, nc, cap);
#pragma unroll 1
    for (int k = 0; k < kRemote; ++k) {
        const uint64_t w = warp_max_u64(mine);
        if (lane == 0) s_cand[warp * kRemote + k] = w;   // 0 when the warp ran out of candidates
        if (mine == w && w != 0) {
            cap = mine;
            mine = best_below(key, tid, kTopkThreads, nc, cap);
        }
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int kPer = kTopkWarps * kRemote / 32;   // survivors per lane
        uint64_t c[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) c[e] = s_cand[lane * kPer + e];
#pragma unroll 1
        for (int k = 0; k < kRemote; ++k) {
            uint64_t best = 0;
            int at = -1;
#pragma unroll
            for (int e = 0; e < kPer; ++e)
                if (c[e] > best) {
                    best = c[e];
                    at = e;
                }
            const uint64_t w = warp_max_u64(best);
            if (best == w && at >= 0) {
#pragma unroll
                for (int e = 0; e < kPer; ++e)
                    if (e == at) c[e] = 0;
            }
            if (lane == 0) out_c[k] = w;
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads)
block_topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
                  const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B,
                  int max_blocks, int32_t *__restrict__ sel, int32_t *dev_err, int staged, int fixed_seq,
                  const uint32_t *__restrict__ cand_mask, int mask_words) {
    extern __shared__ uint32_t s_keys[];
    __shared__ uint64_t s_surv[kSurvivorCap];
    __shared__ uint64_t s_cand[kTopkWarps * kRemote];
    __shared__ uint64_t s_top[kRemote];
    __shared__ uint32_t s_wmax[kTopkWarps];
    __shared__ uint32_t s_thr;
    __shared__ int s_n;
    __shared__ int s_allowed;

    const int i = blockIdx.x;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    int32_t *out = sel + (size_t)i * kSel;

    pdl_wait();
    // the attention kernel of a decode call may start its prologue while this runs
    pdl_launch_dependents();

    QueryRef r;
    if (!resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, tid == 0, r, fixed_seq)) {
        if (tid < kSel) out[tid] = -1;
        return;
    }
    const int nb = r.nb;
    const int nc = nb - kLocal > 0 ? nb - kLocal : 0;
    const uint32_t *mask = cand_mask ? cand_mask + (size_t)r.b * mask_words : nullptr;
    if (nc <= kRemote && !mask) {
        // every causal block fits in the 16 slots
        if (tid < kSel) out[tid] = tid < nb ? tid : -1;
        return;
    }
    const float *row = scores + (size_t)i * max_blocks;
    KeySource key{nullptr, row, mask};
    if (tid == 0) {
        s_n = 0;
        s_allowed = 0;
    }
    __syncthreads();

    // ---- 1. stage keys, 2. per-thread then per-warp maximum
    uint32_t tmax = 0;
    int allowed = 0;
    if (staged) {
#pragma unroll 8
        for (int j = tid; j < nc; j += kTopkThreads) {
            const uint32_t k = key.raw(j);
            s_keys[j] = k;
            tmax = k > tmax ? k : tmax;
            allowed += k != 0u;
        }
        key.smem = s_keys;
    } else {
        for (int j = tid; j < nc; j += kTopkThreads) {
            const uint32_t k = key(j);
            tmax = k > tmax ? k : tmax;
            allowed += k != 0u;
        }
    }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, tmax);
    if (lane == 0) s_wmax[warp] = wmax;
    if (mask) {
        const int wa = __reduce_add_sync(0xffffffffu, allowed);
        if (lane == 0) atomicAdd(&s_allowed, wa);
    }
    __syncthreads();

    if (mask && s_allowed <= kRemote) {
        // no more allowed candidates than remote slots: take them all, in id order
        if (warp == 0) {
            int pos = 0;
            for (int base = 0; base < nc; base += 32) {
                const int j = base + lane;
                const bool take = j < nc && key(j) != 0u;
                const unsigned m = __ballot_sync(0xffffffffu, take);
                if (take) out[pos + __popc(m & ((1u << lane) - 1u))] = j;
                pos += __popc(m);
            }
            const int n_loc = nb < kLocal ? nb : kLocal;
            if (lane < n_loc) out[pos + lane] = nb - n_loc + lane;
            if (lane >= pos + n_loc && lane < kSel) out[lane] = -1;
        }
        return;
    }

    // ---- threshold = the kRemote-th largest warp maximum (with multiplicity)
    if (warp == 0) {
        const uint32_t v = lane < kTopkWarps ? s_wmax[lane] : 0u;
        int gt = 0, ge = 0;
#pragma unroll
        for (int w = 0; w < kTopkWarps; ++w) {
            const uint32_t o = s_wmax[w];
            gt += o > v;
            ge += o >= v;
        }
        const bool is_thr = lane < kTopkWarps && gt <= kRemote - 1 && kRemote - 1 < ge;
        const unsigned who = __ballot_sync(0xffffffffu, is_thr);
        if (lane == __ffs(who) - 1) s_thr = v;
    }
    __syncthreads();
    const uint32_t thr = s_thr;

    // ---- 3. survivors: every candidate at or above the threshold
    for (int j0 = 0; j0 < nc; j0 += kTopkThreads) {
        const int j = j0 + tid;
        const uint32_t k = j < nc ? key(j) : 0u;
        const bool keep = j < nc && k >= thr;
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (m) {
            const int leader = __ffs(m) - 1;
            int base = 0;
            if (lane == leader) base = atomicAdd(&s_n, __popc(m));
            base = __shfl_sync(0xffffffffu, base, leader);
            const int slot = base + __popc(m & ((1u << lane) - 1u));
            if (keep && slot < kSurvivorCap) s_surv[slot] = composite(k, j);
        }
    }
    __syncthreads();
    const int n = s_n;
    if (n <= kSurvivorCap) {
        for (int a = tid; a < n; a += kTopkThreads) {
            const uint64_t c = s_surv[a];
            int rank = 0;
            for (int b = 0; b < n; ++b) rank += s_surv[b] > c;
            if (rank < kRemote) s_top[rank] = c;
        }
        __syncthreads();
    } else {
        topk_two_level(key, nc, s_cand, s_top);
    }

    // ---- 4. the 12 remote ids ascending, then the 4 local blocks
    if (warp == 0) {
        const int id = lane < kRemote ? (int)~(uint32_t)(s_top[lane] & 0xffffffffu) : 0x7fffffff;
        int rank = 0;
#pragma unroll
        for (int k = 0; k < kRemote; ++k) {
            const int other = __shfl_sync(0xffffffffu, id, k);
            rank += other < id;
        }
        if (lane < kRemote) out[rank] = id;
        if (lane < kLocal) out[kRemote + lane] = nb - kLocal + lane;
    }
}

cudaError_t launch_block_topk(const LaunchCtx &c, const float *scores, const int32_t *seq_lens,
                              const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                              int max_blocks, int32_t *sel, int32_t *dev_err, int fixed_seq,
                              const uint32_t *cand_mask, int mask_words) {
    const int staged = max_blocks <= kTopkSmemKeys;
    const size_t smem = staged ? (size_t)max_blocks * sizeof(uint32_t) : 0;
    if (smem > 16 * 1024) {
        // the static shared memory (~19 KiB) plus the staged keys may pass the 48 KiB default
        cudaError_t e = cudaFuncSetAttribute(block_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_q);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, block_topk_kernel, scores, seq_lens, q_seq, q_pos, B, max_blocks,
                              sel, dev_err, staged, fixed_seq, cand_mask, mask_words);
}

}  // namespace uocr
