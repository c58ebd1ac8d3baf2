// index_scan.cu -- Lightning-Indexer block scan for decode queries.
//
// Computes, for every causal 32-token block j of a query at position p,
//   score[j] = max_{t in block j, t <= p} sum_{d<128} idx_q[d] * idx_k[t][d]
// (Unlimited-OCR-2 walk-through, news.rkmt.cn/news/25027, section 五 steps 1-2:
// one indexer head of 128 dims, block score = max over the block's tokens).
//
// Roofline: HBM-bound streaming.  Every causal indexer page (8 KiB) is read
// once; 4 bytes of score are written per page.  Design:
//   * one warp per page: 16 coalesced 16-byte loads per lane cover the page
//     (lane l, step s holds token 2s + l/16, dims 8*(l%16) .. +8);
//   * 8 fp32 FMAs per load against the lane's 8 query dims (kept in registers);
//   * a 15-shuffle transposed reduction leaves each lane with one full token
//     dot product, then a 5-shuffle warp max gives the block score;
//   * loads bypass L1 allocation; 32 warps per SM (4 CTAs of 8) keep the HBM busy.
// The grid is flat over (query, chunk of pages); chunks past a query's causal
// blocks exit at once, so ragged batches need no host-side work list.

#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "scan_core.cuh"

namespace uocr {

constexpr int kScanWarps = 8;

// (256, 4): 64 registers, 4 CTAs x 8 warps per SM (2 CTAs at 96 registers and 5 at 48 are slower)
__global__ void __launch_bounds__(kScanWarps * 32, 4)
index_scan_kernel(const uint4 *__restrict__ idx_q, const uint4 *__restrict__ idx_k,
                  const int32_t *__restrict__ bt, const int32_t *__restrict__ seq_lens,
                  const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B,
                  int max_blocks, int num_pages, int pages_per_warp, int n_chunks,
                  float *__restrict__ scores, int32_t *dev_err) {
    const int i = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x - i * n_chunks;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_wait();

    QueryRef r;
    if (!resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err,
                       chunk == 0 && threadIdx.x == 0, r))
        return;
    const int j0 = chunk * kScanWarps * pages_per_warp;
    if (j0 >= r.nb) return;

    float qf[8];
    bf16x8_to_f32(__ldg(idx_q + (size_t)i * (kDIdx / 8) + (lane & 15)), qf);

    const int j_end = min(r.nb, j0 + kScanWarps * pages_per_warp);
    scan_pages(qf, idx_k, bt + (size_t)r.b * max_blocks, r.p, j0 + warp, kScanWarps, j_end, num_pages,
               scores + (size_t)i * max_blocks, dev_err, lane);
    pdl_launch_dependents();
}

cudaError_t launch_index_scan(const LaunchCtx &c, const void *idx_q, const void *idx_k,
                              const int32_t *bt, const int32_t *seq_lens, const int32_t *q_seq,
                              const int32_t *q_pos, int n_q, int B, int max_blocks, int num_pages,
                              float *scores, int32_t *dev_err) {
    // Pages per warp: enough CTAs for ~16 waves of 4 CTAs per SM, at most 8 pages per warp.
    const long long total_pages = (long long)n_q * max_blocks;
    const long long target_ctas = 16LL * c.num_sms * 4;
    long long ppw = total_pages / (target_ctas * kScanWarps);
    if (ppw < 1) ppw = 1;
    if (ppw > 8) ppw = 8;
    const int pages_per_cta = kScanWarps * (int)ppw;
    const int n_chunks = (max_blocks + pages_per_cta - 1) / pages_per_cta;
    const long long grid = (long long)n_chunks * n_q;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kScanWarps * 32);
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, index_scan_kernel, (const uint4 *)idx_q, (const uint4 *)idx_k, bt,
                              seq_lens, q_seq, q_pos, B, max_blocks, num_pages, (int)ppw, n_chunks,
                              scores, dev_err);
}

}  // namespace uocr

