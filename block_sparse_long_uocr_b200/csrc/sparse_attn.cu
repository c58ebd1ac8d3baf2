// sparse_attn.cu -- exact attention over the selected 16 x 32 tokens.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 step 4:
// attention runs over only the selected blocks (16 blocks x 32 tokens = 512
// tokens per query), never materialising a full score row; section 三: MHA
// with 10 heads of 128 dims.  Per head h of query i at position p:
//   z_t = scale * q . k_t  (t <= p in the selected blocks),
//   out = sum_t softmax(z)_t v_t      (fp32 softmax and accumulation).
//
// Split-K (flash-decoding): CTA (i, h, s) handles 4 of the 16 selected blocks,
// one warp per block.  A warp streams the block's K tile (8 KiB) and V tile
// (8 KiB) with coalesced 16-byte loads: for step t lane l holds token
// 2t + l/16, dims 8*(l%16) .. +8.  Scores come from a transposed half-warp
// reduction (each lane ends with one token), the block's (max, sum, acc[128])
// softmax state is merged across the 4 warps in shared memory and written to
// the workspace; a second kernel merges the splits and writes bf16.
// Roofline: HBM-bound, 2 x 8 KiB per (block, head), no reuse across queries.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

constexpr int kAttnWarps = 4;             // blocks per CTA (one per warp)
constexpr int kAttnSplits = kSel / kAttnWarps;

int attn_splits(int, int) { return kAttnSplits; }

__global__ void __launch_bounds__(kAttnWarps * 32)
sparse_attn_split_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ kc,
                         const uint4 *__restrict__ vc, const int32_t *__restrict__ bt,
                         const int32_t *__restrict__ seq_lens, const int32_t *__restrict__ q_seq,
                         const int32_t *__restrict__ q_pos, const int32_t *__restrict__ sel, int B,
                         int H, int max_blocks, int num_pages, float scale_log2,
                         float *__restrict__ part_acc, float *__restrict__ part_ml,
                         int32_t *dev_err) {
    __shared__ float s_m[kAttnWarps], s_l[kAttnWarps];
    __shared__ float s_acc[kAttnWarps][kD];

    const int split = blockIdx.x % kAttnSplits;
    const int ih = blockIdx.x / kAttnSplits;
    const int h = ih % H;
    const int i = ih / H;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_wait();

    float m_w = -INFINITY, l_w = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    QueryRef r;
    const bool ok = resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err,
                                  threadIdx.x == 0 && split == 0 && h == 0, r);
    const int j = ok ? __ldg(sel + (size_t)i * kSel + split * kAttnWarps + warp) : -1;
    int page = -1;
    if (j >= 0) {
        if (j >= r.nb) {
            if (lane == 0) flag_error(dev_err, UOCR_DEVERR_SEL);
        } else {
            page = __ldg(bt + (size_t)r.b * max_blocks + j);
            if ((unsigned)page >= (unsigned)num_pages) {
                if (lane == 0) flag_error(dev_err, UOCR_DEVERR_PAGE);
                page = -1;
            }
        }
    }

    if (page >= 0) {
        float qf[8];
        bf16x8_to_f32(__ldg(q + ((size_t)i * H + h) * (kD / 8) + (lane & 15)), qf);
        const size_t tile = ((size_t)page * H + h) * (kPageElems / 8) + lane;

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
            for (int e = 1; e < 8; ++e) a = fmaf(qf[e], kf[e], a);
            z[t] = a;
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) kv[t] = ld_stream(vc + tile + t * 32);

        // lane now owns token 2*(lane&15) + lane/16 of the block
        float zt = half_warp_transpose_sum16(z, lane) * scale_log2;
        const int tok = 2 * (lane & 15) + (lane >> 4);
        if (j * kBlock + tok > r.p) zt = -INFINITY;
        m_w = warp_max(zt);                       // finite: token 32j <= p is visible
        const float pt = exp2f(zt - m_w);
        l_w = warp_sum(pt);

#pragma unroll
        for (int t = 0; t < 16; ++t) {
            // weight of token 2t + lane/16, owned by lane (lane & 16) | t
            const float w = __shfl_sync(0xffffffffu, pt, (lane & 16) | t);
            float vf[8];
            bf16x8_to_f32(kv[t], vf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, vf[e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    }

    if (lane == 0) {
        s_m[warp] = m_w;
        s_l[warp] = l_w;
    }
    if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s_acc[warp][lane * 8 + e] = acc[e];
    }
    __syncthreads();

    // merge the 4 warps' softmax states; thread d owns output dim d
    const int d = threadIdx.x;
    float M = s_m[0];
#pragma unroll
    for (int w = 1; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float f = exp2f(s_m[w] - M);   // 0 for an empty warp (m = -inf)
            L = fmaf(s_l[w], f, L);
            A = fmaf(s_acc[w][d], f, A);
        }
    }
    const size_t slot = (size_t)blockIdx.x;     // ((i*H + h)*kAttnSplits + split)
    part_acc[slot * kD + d] = A;
    if (d == 0) {
        part_ml[slot * 2] = M;
        part_ml[slot * 2 + 1] = L;
    }
    pdl_launch_dependents();
}

__global__ void __launch_bounds__(kD)
sparse_attn_combine_kernel(const float *__restrict__ part_acc, const float *__restrict__ part_ml,
                           __nv_bfloat16 *__restrict__ out) {
    const int ih = blockIdx.x;
    const int d = threadIdx.x;
    pdl_wait();
    const float *ml = part_ml + (size_t)ih * kAttnSplits * 2;
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kAttnSplits; ++s) M = fmaxf(M, ml[2 * s]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int s = 0; s < kAttnSplits; ++s) {
            const float f = exp2f(ml[2 * s] - M);
            L = fmaf(ml[2 * s + 1], f, L);
            A = fmaf(part_acc[((size_t)ih * kAttnSplits + s) * kD + d], f, A);
        }
    }
    out[(size_t)ih * kD + d] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
    pdl_launch_dependents();
}

cudaError_t launch_sparse_attn(const LaunchCtx &c, const void *q, const void *k, const void *v,
                               const int32_t *bt, const int32_t *seq_lens, const int32_t *q_seq,
                               const int32_t *q_pos, const int32_t *sel, int n_q, int B, int H,
                               int max_blocks, int num_pages, float scale, void *out,
                               float *part_acc, float *part_ml, int32_t *dev_err) {
    const long long grid = (long long)n_q * H * kAttnSplits;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kAttnWarps * 32);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, sparse_attn_split_kernel, (const uint4 *)q,
                                       (const uint4 *)k, (const uint4 *)v, bt, seq_lens, q_seq,
                                       q_pos, sel, B, H, max_blocks, num_pages, scale * kLog2e,
                                       part_acc, part_ml, dev_err);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg2 = {};
    cfg2.gridDim = dim3((unsigned)(n_q * H));
    cfg2.blockDim = dim3(kD);
    cfg2.stream = c.stream;
    cfg2.attrs = attr;
    cfg2.numAttrs = 1;   // always a dependent of the split kernel
    return cudaLaunchKernelEx(&cfg2, sparse_attn_combine_kernel, (const float *)part_acc,
                              (const float *)part_ml, (__nv_bfloat16 *)out);
}

}  // namespace uocr
