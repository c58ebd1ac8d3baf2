// scan_core.cuh -- one query's indexer scan over a set of pages (a warp per page).
//
// Block score of the walk-through (news.rkmt.cn/news/25027, section 五 step 2):
//   score[j] = max_{t in block j, t <= p} sum_{d<128} idx_q[d] * idx_k[t][d].
// A warp reads one 8 KiB page with 16 coalesced 16-byte loads per lane (step s:
// lane l holds token 2s + l/16, dims 8*(l%16) .. +8), does 8 fp32 FMAs per load
// against the lane's 8 query dims, reduces with the 15-shuffle transposed
// half-warp sum (each lane ends with one token's dot product) and a 5-shuffle
// warp max.  attend_block_online is the per-block online-softmax step of the
// comparator decode attention (dense_attn.cu).
#pragma once

#include "common.cuh"

namespace uocr {

// Scores of pages j = j_first, j_first + j_step, ... < j_end of one query; called by a whole warp.
__device__ __forceinline__ void scan_pages(const float (&qf)[8], const uint4 *__restrict__ idx_k,
                                           const int32_t *__restrict__ bt_row, int p, int j_first, int j_step,
                                           int j_end, int num_pages, float *__restrict__ srow, int32_t *dev_err,
                                           int lane) {
    const int tok = 2 * (lane & 15) + (lane >> 4);
    for (int j = j_first; j < j_end; j += j_step) {
        const int page = __ldg(bt_row + j);
        if ((unsigned)page >= (unsigned)num_pages) {
            if (lane == 0) {
                flag_error(dev_err, UOCR_DEVERR_PAGE);
                srow[j] = -INFINITY;
            }
            continue;
        }
        const uint4 *src = idx_k + (size_t)page * (kBlock * kDIdx / 8) + lane;
        uint4 v[16];
#pragma unroll
        for (int s = 0; s < 16; ++s) v[s] = ld_stream(src + s * 32);
        float acc[16];
#pragma unroll
        for (int s = 0; s < 16; ++s) {
            float kf[8];
            bf16x8_to_f32(v[s], kf);
            float a = qf[0] * kf[0];
#pragma unroll
            for (int e = 1; e < 8; ++e) a = fmaf(qf[e], kf[e], a);
            acc[s] = a;
        }
        float dot = half_warp_transpose_sum16(acc, lane);
        if (j * kBlock + tok > p) dot = -INFINITY;
        const float m = warp_max(dot);
        if (lane == 0) srow[j] = m;
    }
}

// One selected (or attended) block of one head, merged into a warp's running softmax state
// (m, l, acc[8]): K and V tiles read through registers, exp2-based fp32 softmax.  After the
// last block the caller adds acc across the two half-warps (lanes l and l^16).
__device__ __forceinline__ void attend_block_online(const float (&qf)[8], const uint4 *__restrict__ kc,
                                                    const uint4 *__restrict__ vc, size_t tile, int j, int p,
                                                    float scale_log2, int lane, float &m_w, float &l_w,
                                                    float (&acc)[8]) {
    const int tok = 2 * (lane & 15) + (lane >> 4);
    uint4 kv[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) kv[t] = ld_stream(kc + tile + t * 32);
    float z[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        float kf[8];
        bf16x8_to_f32(kv[t], kf);
        float a = qf[0] * kf[0];
#pragma unroll
        for (int c = 1; c < 8; ++c) a = fmaf(qf[c], kf[c], a);
        z[t] = a;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) kv[t] = ld_stream(vc + tile + t * 32);
    float zt = half_warp_transpose_sum16(z, lane) * scale_log2;
    if (j * kBlock + tok > p) zt = -INFINITY;
    const float mb = warp_max(zt);                  // finite: token 32j <= p
    const float m_new = fmaxf(m_w, mb);
    const float corr = exp2f(m_w - m_new);          // 0 on the first block (m_w = -inf)
    const float pt = exp2f(zt - m_new);
    l_w = l_w * corr + warp_sum(pt);
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= corr;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const float w = __shfl_sync(0xffffffffu, pt, (lane & 16) | t);
        float vf[8];
        bf16x8_to_f32(kv[t], vf);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(w, vf[c], acc[c]);
    }
    m_w = m_new;
}

}  // namespace uocr
