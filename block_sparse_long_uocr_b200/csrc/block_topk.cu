// block_topk.cu -- per-query block selection: 4 local blocks + top-12 remote.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 step 3:
// each query keeps 16 blocks, the 4 most recent ("local", the 128-token
// window) and the 12 remote blocks with the highest indexer score; inference
// uses a hard top-k.  Ranking: score descending, then lower block id.
//
// One CTA per query.  The 12th-largest score is found exactly by a 4-pass,
// 8-bit radix select on order-preserving fp32 keys (shared-memory histograms),
// then one ordered pass over contiguous per-thread id ranges emits the chosen
// remote ids in ascending order, taking the lowest ids among keys equal to the
// threshold.  Cost is ~5 reads of the candidate scores from L2 per query.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

constexpr int kTopkThreads = 256;

// Larger key <=> larger float (total order on non-NaN values, -0 < +0).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA; also returns the total through *total.
__device__ __forceinline__ int cta_exclusive_scan(int x, int *warp_buf, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_buf[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kTopkThreads / 32 ? warp_buf[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kTopkThreads / 32) warp_buf[lane] = wi - w;
        if (lane == kTopkThreads / 32 - 1) warp_buf[kTopkThreads / 32] = wi;
    }
    __syncthreads();
    const int res = warp_buf[warp] + incl - x;
    *total = warp_buf[kTopkThreads / 32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kTopkThreads)
block_topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
                  const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B,
                  int max_blocks, int32_t *__restrict__ sel, int32_t *dev_err) {
    __shared__ int hist[256];
    __shared__ int warp_buf[kTopkThreads / 32 + 1];
    __shared__ uint32_t s_prefix;
    __shared__ int s_need;

    const int i = blockIdx.x;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    int32_t *out = sel + (size_t)i * kSel;

    pdl_wait();
    QueryRef r;
    if (!resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, tid == 0, r)) {
        if (tid < kSel) out[tid] = -1;
        return;
    }
    const int nb = r.nb;
    const int nc = nb - kLocal > 0 ? nb - kLocal : 0;
    if (nc <= kRemote) {
        // every causal block fits in the 16 slots
        if (tid < kSel) out[tid] = tid < nb ? tid : -1;
        return;
    }
    const float *s = scores + (size_t)i * max_blocks;

    // ---- radix select of the kRemote-th largest key
    uint32_t prefix = 0, mask = 0;
    int need = kRemote;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = tid; b < 256; b += kTopkThreads) hist[b] = 0;
        __syncthreads();
        for (int j = tid; j < nc; j += kTopkThreads) {
            const uint32_t key = order_key(s[j]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane L owns bins 255-8L .. 248-8L (descending); find the bin holding rank `need`
            int c[8], tot = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                c[k] = hist[255 - 8 * lane - k];
                tot += c[k];
            }
            int incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            const int excl = incl - tot;
            const unsigned owner = __ballot_sync(0xffffffffu, excl < need && need <= incl);
            if (lane == __ffs(owner) - 1) {
                int run = excl;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (run + c[k] >= need) {
                        s_prefix = prefix | ((uint32_t)(255 - 8 * lane - k) << shift);
                        s_need = need - run;
                        break;
                    }
                    run += c[k];
                }
            }
        }
        __syncthreads();
        prefix = s_prefix;
        need = s_need;
        mask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t thr = prefix;   // key of the kRemote-th ranked candidate
    // `need` = how many candidates equal to thr are taken (the lowest ids among them)

    // ---- ordered emission over contiguous id ranges
    const int per = (nc + kTopkThreads - 1) / kTopkThreads;
    const int lo = tid * per;
    const int hi = lo + per < nc ? lo + per : nc;
    int n_eq = 0;
    for (int j = lo; j < hi; ++j) n_eq += order_key(s[j]) == thr;
    int total;
    const int eq_base = cta_exclusive_scan(n_eq, warp_buf, &total);
    int n_take = 0;
    {
        int seen = eq_base;
        for (int j = lo; j < hi; ++j) {
            const uint32_t key = order_key(s[j]);
            const bool eq = key == thr;
            n_take += (key > thr) || (eq && seen < need);
            seen += eq;
        }
    }
    const int pos0 = cta_exclusive_scan(n_take, warp_buf, &total);
    {
        int seen = eq_base, pos = pos0;
        for (int j = lo; j < hi; ++j) {
            const uint32_t key = order_key(s[j]);
            const bool eq = key == thr;
            if ((key > thr) || (eq && seen < need)) {
                if (pos < kRemote) out[pos] = j;
                ++pos;
            }
            seen += eq;
        }
    }
    if (tid < kLocal) out[kRemote + tid] = nb - kLocal + tid;
    pdl_launch_dependents();
}

cudaError_t launch_block_topk(const LaunchCtx &c, const float *scores, const int32_t *seq_lens,
                              const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                              int max_blocks, int32_t *sel, int32_t *dev_err) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_q);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, block_topk_kernel, scores, seq_lens, q_seq, q_pos, B, max_blocks,
                              sel, dev_err);
}

}  // namespace uocr
