// block_topk.cu -- per-query block selection: 4 local blocks + top-12 remote.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 step 3:
// each query keeps 16 blocks, the 4 most recent ("local", the 128-token
// window) and the 12 remote blocks with the highest indexer score; inference
// uses a hard top-k.  Ranking: score descending, then lower block id.
//
// One CTA of 512 threads per query runs topk_select (topk_core.cuh): scores
// staged in shared memory, a threshold from 16 warp maxima, survivors ranked by
// counting, an exact two-level fallback for heavily tied rows, and an optional
// page-aware candidate bitmap (section 五 image_bucket_constraint).  Rows longer
// than the shared-memory budget are read from L2 instead of staged.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "topk_core.cuh"

namespace uocr {

constexpr int kTopkThreads = 512;
constexpr int kTopkSmemKeys = 48 * 1024;    // stage rows up to 48K candidates (192 KiB of keys)

__global__ void __launch_bounds__(kTopkThreads)
block_topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
                  const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B,
                  int max_blocks, int32_t *__restrict__ sel, int32_t *dev_err, int staged, int fixed_seq,
                  const uint32_t *__restrict__ cand_mask, int mask_words) {
    extern __shared__ uint32_t s_keys[];
    __shared__ TopkShared<kTopkThreads> sm;
    const int i = blockIdx.x;
    const int tid = threadIdx.x;
    int32_t *out = sel + (size_t)i * kSel;

    pdl_wait();
    // the attention kernel of a decode call may start its prologue while this runs
    pdl_launch_dependents();

    QueryRef r;
    if (!resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, tid == 0, r, fixed_seq)) {
        if (tid < kSel) out[tid] = -1;
        return;
    }
    const uint32_t *mask = cand_mask ? cand_mask + (size_t)r.b * mask_words : nullptr;
    topk_select<kTopkThreads>(scores + (size_t)i * max_blocks, r.nb, mask, staged ? s_keys : nullptr, sm, out);
}

cudaError_t launch_block_topk(const LaunchCtx &c, const float *scores, const int32_t *seq_lens,
                              const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                              int max_blocks, int32_t *sel, int32_t *dev_err, int fixed_seq,
                              const uint32_t *cand_mask, int mask_words) {
    const int staged = max_blocks <= kTopkSmemKeys;
    const size_t smem = staged ? (size_t)max_blocks * sizeof(uint32_t) : 0;
    if (smem > 16 * 1024) {
        // the static shared memory (~18 KiB) plus the staged keys may pass the 48 KiB default
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
