// block_topk.cu -- per-query block selection: 4 local blocks + top-12 remote.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 step 3:
// each query keeps 16 blocks, the 4 most recent ("local", the 128-token
// window) and the 12 remote blocks with the highest indexer score; inference
// uses a hard top-k.  Ranking: score descending, then lower block id.
//
// Few rows (decode): one CTA of 512 threads per query runs topk_select
// (topk_core.cuh): keys in registers (rows of up to 4096 candidates) or staged
// in shared memory, a threshold from 16 warp maxima, survivors ranked by
// counting, an exact two-level fallback for heavily tied rows, and an optional
// page-aware candidate bitmap (section 五 image_bucket_constraint).  Rows longer
// than the shared-memory budget are read from L2 instead of staged.  Many rows (a prefill chunk): one warp per query
// runs topk_warp_select, the same steps at warp scope, so that every row is in
// flight at once.  Either kernel can also count, per block, the queries that
// selected it (the first step of the block-centric prefill attention).
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "topk_core.cuh"

namespace uocr {

constexpr int kTopkThreads = 512;
constexpr int kTopkSmemKeys = 48 * 1024;    // stage rows up to 48K candidates (192 KiB of keys)
constexpr int kTopkWarpRows = 14;           // queries (warps) per CTA of the warp-per-row kernel: 2048 rows fill 147 SMs evenly
constexpr int kWarpRowsFrom = 512;          // use the warp-per-row kernel from this many queries

// counts[v] += 1 for every selected block v of one query's 16 slots (lanes 0..15 of the caller).
__device__ __forceinline__ void count_selected(const int32_t *out, int slot, int32_t *counts) {
    const int v = out[slot];
    if (v >= 0) atomicAdd(counts + v, 1);
}

// (512, 1): without the block count ptxas fits 4 CTAs per SM in 32 registers and spills
__global__ void __launch_bounds__(kTopkThreads, 1)
block_topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
                  const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B,
                  int max_blocks, int32_t *__restrict__ sel, int32_t *dev_err, int staged, int fixed_seq,
                  const uint32_t *__restrict__ cand_mask, int mask_words, int32_t *counts) {
    extern __shared__ uint32_t s_keys[];
    __shared__ TopkShared<kTopkThreads> sm;
    const int i = blockIdx.x;
    const int tid = threadIdx.x;
    int32_t *out = sel + (size_t)i * kSel;

    // the query's metadata are inputs of the call, not outputs of the preceding kernel
    QueryRef r;
    const bool ok = resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, tid == 0, r, fixed_seq);
    pdl_wait();
    // the attention kernel of a decode call may start its prologue while this runs
    pdl_launch_dependents();
    if (!ok) {
        if (tid < kSel) out[tid] = -1;
        return;
    }
    const uint32_t *mask = cand_mask ? cand_mask + (size_t)r.b * mask_words : nullptr;
    topk_select<kTopkThreads>(scores + (size_t)i * max_blocks, r.nb, mask, staged ? s_keys : nullptr, sm, out);
    if (counts) {
        __syncthreads();
        if (tid < kSel) count_selected(out, tid, counts);
    }
}

__global__ void __launch_bounds__(kTopkWarpRows * 32)
block_topk_warp_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
                       const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B, int n_q,
                       int max_blocks, int32_t *__restrict__ sel, int32_t *dev_err, int fixed_seq,
                       const uint32_t *__restrict__ cand_mask, int mask_words, int32_t *counts) {
    __shared__ TopkWarpShared sm[kTopkWarpRows];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * kTopkWarpRows + warp;
    pdl_wait();
    // No early trigger: this grid holds nearly every SM's registers while it runs, so a dependent
    // grid launched early would crowd its CTAs onto the few SMs left free.  Each warp lets the
    // dependents start once its row is done (the grid triggers when every warp has, or exited).
    if (i >= n_q) return;
    int32_t *out = sel + (size_t)i * kSel;
    QueryRef r;
    if (!resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, lane == 0, r, fixed_seq)) {
        if (lane < kSel) out[lane] = -1;
        return;
    }
    const uint32_t *mask = cand_mask ? cand_mask + (size_t)r.b * mask_words : nullptr;
    topk_warp_select(scores + (size_t)i * max_blocks, r.nb, mask, sm[warp], out);
    if (counts) {
        __syncwarp();
        if (lane < kSel) count_selected(out, lane, counts);
    }
    pdl_launch_dependents();
}

cudaError_t launch_block_topk(const LaunchCtx &c, const float *scores, const int32_t *seq_lens,
                              const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                              int max_blocks, int32_t *sel, int32_t *dev_err, int fixed_seq,
                              const uint32_t *cand_mask, int mask_words, int32_t *counts) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (n_q >= kWarpRowsFrom) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((n_q + kTopkWarpRows - 1) / kTopkWarpRows));
        cfg.blockDim = dim3(kTopkWarpRows * 32);
        cfg.stream = c.stream;
        cfg.attrs = attr;
        cfg.numAttrs = c.pdl ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, block_topk_warp_kernel, scores, seq_lens, q_seq, q_pos, B, n_q, max_blocks,
                                  sel, dev_err, fixed_seq, cand_mask, mask_words, counts);
    }
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
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, block_topk_kernel, scores, seq_lens, q_seq, q_pos, B, max_blocks,
                              sel, dev_err, staged, fixed_seq, cand_mask, mask_words, counts);
}

}  // namespace uocr
