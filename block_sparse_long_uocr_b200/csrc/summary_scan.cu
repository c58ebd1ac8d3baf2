// summary_scan.cu -- block-summary indexer scoring and the mean-key summary.
//
// The pages also describe the coarse screen as scoring each KV block through a
// summary: "learnable summary vectors" per block (Unlimited-OCR-2-8bit page,
// www.lqnn.cn/news/271890, section 显存账本) and a block's "brief
// representation" before reading its tokens (release report, leheavengame.com,
// section 二, Token Sieve).  This variant scores causal block j of a query by
//   s[j] = idx_q . summary[block_table[b][j]]
// with one bf16 summary vector (128 dims, 256 bytes) per page instead of the
// page's 32 indexer keys: 32x fewer bytes than the max-over-tokens scan.  The
// summaries are an input (a trained model supplies them); block_mean_kernel
// builds the simplest untrained one, the mean of the page's 32 indexer keys.
//
// Scan layout: a half-warp per page (16 lanes x 16 bytes = one summary), 8 fp32
// FMAs per lane and a 4-shuffle reduction, 8 pages per half-warp in flight; the
// grid is flat over (query, chunk of pages) like the token scan.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

namespace {
constexpr int kSumWarps = 8;
constexpr int kSumBatch = 8;   // pages per half-warp whose loads are in flight together
}  // namespace

__global__ void __launch_bounds__(kSumWarps * 32)
summary_scan_kernel(const uint4 *__restrict__ idx_q, const uint4 *__restrict__ summary,
                    const int32_t *__restrict__ bt, const int32_t *__restrict__ seq_lens,
                    const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos, int B, int max_blocks,
                    int num_pages, int pages_per_cta, int n_chunks, float *__restrict__ scores, int32_t *dev_err) {
    const int i = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x - i * n_chunks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    pdl_wait();
    QueryRef r;
    if (!resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, chunk == 0 && threadIdx.x == 0, r)) return;
    const int j0 = chunk * pages_per_cta;
    if (j0 >= r.nb) return;
    float qf[8];
    bf16x8_to_f32(__ldg(idx_q + (size_t)i * (kDIdx / 8) + hl), qf);
    const int32_t *bt_row = bt + (size_t)r.b * max_blocks;
    float *srow = scores + (size_t)i * max_blocks;
    const int jend = min(r.nb, j0 + pages_per_cta);
    // A half-warp's pages are jw + half, + 16, ..., kSumBatch at a time: all block-table loads
    // issued, then all summary loads, then the math, so that the two dependent round trips are
    // paid once per batch instead of once per page.  The loop bound is the warp's (the same for
    // both half-warps).
    for (int jw = j0 + warp * 2; jw < jend; jw += kSumBatch * kSumWarps * 2) {
        const int jb = jw + half;
        int page[kSumBatch];
#pragma unroll
        for (int k = 0; k < kSumBatch; ++k) {
            const int j = jb + k * kSumWarps * 2;
            page[k] = j < jend ? __ldg(bt_row + j) : -1;
        }
        uint4 v[kSumBatch];
#pragma unroll
        for (int k = 0; k < kSumBatch; ++k)
            v[k] = (unsigned)page[k] < (unsigned)num_pages ? ld_stream(summary + (size_t)page[k] * (kDIdx / 8) + hl)
                                                          : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < kSumBatch; ++k) {
            const int j = jb + k * kSumWarps * 2;
            float kf[8];
            bf16x8_to_f32(v[k], kf);
            float a = qf[0] * kf[0];
#pragma unroll
            for (int c = 1; c < 8; ++c) a = fmaf(qf[c], kf[c], a);
            // both half-warps run the same iterations (j past jend only idles), so the whole warp
            // takes part in every shuffle
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (hl == 0 && j < jend) {
                const bool ok = (unsigned)page[k] < (unsigned)num_pages;
                if (!ok) flag_error(dev_err, UOCR_DEVERR_PAGE);
                srow[j] = ok ? a : -INFINITY;
            }
        }
    }
    pdl_launch_dependents();
}

// summary[page] = bf16(mean of the page's 32 indexer keys), one warp per page (lane: 4 dims).
__global__ void __launch_bounds__(256)
block_mean_kernel(const __nv_bfloat16 *__restrict__ idx_k, const int32_t *__restrict__ pages, int n_pages,
                  int num_pages, __nv_bfloat16 *__restrict__ summary, int32_t *dev_err) {
    const int w = (blockIdx.x * 256 + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    if (w >= n_pages) return;
    const int page = pages ? __ldg(pages + w) : w;
    if ((unsigned)page >= (unsigned)num_pages) {
        if (lane == 0) flag_error(dev_err, UOCR_DEVERR_PAGE);
        return;
    }
    const uint2 *src = reinterpret_cast<const uint2 *>(idx_k + (size_t)page * kBlock * kDIdx) + lane;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int r = 0; r < kBlock; ++r) {
        const uint2 v = __ldg(src + r * (kDIdx / 4));
        acc[0] += __uint_as_float(v.x << 16);
        acc[1] += __uint_as_float(v.x & 0xffff0000u);
        acc[2] += __uint_as_float(v.y << 16);
        acc[3] += __uint_as_float(v.y & 0xffff0000u);
    }
    __nv_bfloat16 *dst = summary + (size_t)page * kDIdx + lane * 4;
#pragma unroll
    for (int c = 0; c < 4; ++c) dst[c] = __float2bfloat16_rn(acc[c] * (1.0f / kBlock));
}

cudaError_t launch_summary_scan(const LaunchCtx &c, const void *idx_q, const void *summary, const int32_t *bt,
                                const int32_t *seq_lens, const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                                int max_blocks, int num_pages, float *scores, int32_t *dev_err) {
    const int pages_per_cta = 256;   // 16 pages per warp
    const int n_chunks = (max_blocks + pages_per_cta - 1) / pages_per_cta;
    const long long grid = (long long)n_chunks * n_q;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kSumWarps * 32);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, summary_scan_kernel, (const uint4 *)idx_q, (const uint4 *)summary, bt, seq_lens,
                              q_seq, q_pos, B, max_blocks, num_pages, pages_per_cta, n_chunks, scores, dev_err);
}

cudaError_t launch_block_mean(const LaunchCtx &c, const void *idx_k, const int32_t *pages, int n_pages,
                              int num_pages, void *summary, int32_t *dev_err) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n_pages + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = c.stream;
    return cudaLaunchKernelEx(&cfg, block_mean_kernel, (const __nv_bfloat16 *)idx_k, pages, n_pages, num_pages,
                              (__nv_bfloat16 *)summary, dev_err);
}

}  // namespace uocr
