// dense_attn.cu -- comparator decode attention: a reference prefix plus the local window.
//
// The pages quote the sparse step's speed against two baselines: full causal
// attention and the previous generation's R-SWA (release report,
// leheavengame.com, section 一: 7.0x and 5.6x per decode step).  R-SWA (Unlimited
// OCR v1 article, chenxutan.com/d/4261.html, section 2.3.2) keeps the reference
// tokens always visible and only a 128-token window of generated tokens.  Both
// are exact attention over a contiguous set of blocks:
//   attended blocks of a query with nb causal blocks =
//       [0, min(ref_blocks, nb))  U  [max(nb - 4, 0), nb)        (t <= p inside)
// ref_blocks >= nb gives full causal attention; a smaller prefix gives R-SWA.
//
// Split-K flash decoding: CTA (query, head, chunk of 16 blocks), 4 warps, warp w
// takes blocks w, w+4, w+8, w+12 of the chunk with an online softmax; the warps
// merge in shared memory into the chunk's partial state (m, l, acc[128]); a
// second kernel merges the chunks of each (query, head).  HBM-bound: every
// attended (block, head) K and V tile (2 x 8 KiB) is read once.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "scan_core.cuh"

namespace uocr {

namespace {
constexpr int kDWarps = 4;
constexpr int kChunkBlocks = 16;
}  // namespace

int dense_chunks(int max_blocks) { return (max_blocks + kChunkBlocks - 1) / kChunkBlocks; }

__device__ __forceinline__ bool dense_attended(int j, int nb, int ref_blocks) {
    return j < nb && (j < ref_blocks || j >= nb - kLocal);
}

__global__ void __launch_bounds__(kDWarps * 32)
dense_attn_chunk_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ kc, const uint4 *__restrict__ vc,
                        const int32_t *__restrict__ bt, const int32_t *__restrict__ seq_lens, int B, int H,
                        int max_blocks, int num_pages, int ref_blocks, int n_chunks, float scale_log2,
                        float *__restrict__ part_acc, float *__restrict__ part_ml, int32_t *dev_err) {
    __shared__ float s_m[kDWarps], s_l[kDWarps];
    __shared__ float s_acc[kDWarps][kD];

    const int chunk = blockIdx.x % n_chunks;
    const int ih = blockIdx.x / n_chunks;
    const int h = ih % H;
    const int i = ih / H;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_wait();
    QueryRef r;
    const bool ok = resolve_query(i, seq_lens, nullptr, nullptr, B, max_blocks, dev_err,
                                  threadIdx.x == 0 && chunk == 0 && h == 0, r);
    const int nb = ok ? r.nb : 0;
    if (chunk * kChunkBlocks >= nb) return;   // the merge reads only the chunks below nb

    float qf[8];
    bf16x8_to_f32(__ldg(q + ((size_t)i * H + h) * (kD / 8) + (lane & 15)), qf);
    float m_w = -INFINITY, l_w = 0.f;
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;

    for (int k = warp; k < kChunkBlocks; k += kDWarps) {
        const int j = chunk * kChunkBlocks + k;
        if (!dense_attended(j, nb, ref_blocks)) continue;
        const int page = __ldg(bt + (size_t)r.b * max_blocks + j);
        if ((unsigned)page >= (unsigned)num_pages) {
            if (lane == 0) flag_error(dev_err, UOCR_DEVERR_PAGE);
            continue;
        }
        attend_block_online(qf, kc, vc, ((size_t)page * H + h) * (kPageElems / 8) + lane, j, r.p, scale_log2,
                            lane, m_w, l_w, acc);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 16);

    if (lane == 0) {
        s_m[warp] = m_w;
        s_l[warp] = l_w;
    }
    if (lane < 16) {
#pragma unroll
        for (int c = 0; c < 8; ++c) s_acc[warp][lane * 8 + c] = acc[c];
    }
    __syncthreads();
    const int d = threadIdx.x;
    float M = s_m[0];
#pragma unroll
    for (int w = 1; w < kDWarps; ++w) M = fmaxf(M, s_m[w]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kDWarps; ++w) {
            const float f = exp2f(s_m[w] - M);
            L = fmaf(s_l[w], f, L);
            A = fmaf(s_acc[w][d], f, A);
        }
    }
    const size_t slot = (size_t)ih * n_chunks + chunk;
    part_acc[slot * kD + d] = A;
    if (d == 0) {
        part_ml[slot * 2] = M;
        part_ml[slot * 2 + 1] = L;
    }
}

__global__ void __launch_bounds__(kD)
dense_attn_merge_kernel(const int32_t *__restrict__ seq_lens, int B, int H, int max_blocks, int n_chunks,
                        const float *__restrict__ part_acc, const float *__restrict__ part_ml,
                        __nv_bfloat16 *__restrict__ out) {
    const int ih = blockIdx.x;
    const int i = ih / H;
    const int d = threadIdx.x;
    pdl_wait();
    QueryRef r;
    const bool ok = resolve_query(i, seq_lens, nullptr, nullptr, B, max_blocks, nullptr, false, r);
    const int used = ok ? (r.nb + kChunkBlocks - 1) / kChunkBlocks : 0;
    float M = -INFINITY;
    for (int c = 0; c < used; ++c) M = fmaxf(M, part_ml[((size_t)ih * n_chunks + c) * 2]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
        for (int c = 0; c < used; ++c) {
            const size_t slot = (size_t)ih * n_chunks + c;
            const float f = exp2f(part_ml[slot * 2] - M);
            L = fmaf(part_ml[slot * 2 + 1], f, L);
            A = fmaf(part_acc[slot * kD + d], f, A);
        }
    }
    out[(size_t)ih * kD + d] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
}

size_t dense_attn_workspace(int n_q, int H, int max_blocks) {
    const size_t slots = (size_t)n_q * H * dense_chunks(max_blocks);
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return up(slots * kD * 4) + up(slots * 2 * 4);
}

cudaError_t launch_dense_attn(const LaunchCtx &c, const void *q, const void *k, const void *v, const int32_t *bt,
                              const int32_t *seq_lens, int B, int H, int max_blocks, int num_pages, int ref_blocks,
                              float scale, void *out, void *ws, int32_t *dev_err) {
    const int n_chunks = dense_chunks(max_blocks);
    const size_t slots = (size_t)B * H * n_chunks;
    float *acc = (float *)ws;
    float *ml = (float *)((char *)ws + (slots * kD * 4 + 255) / 256 * 256);
    const long long grid = (long long)slots;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kDWarps * 32);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, dense_attn_chunk_kernel, (const uint4 *)q, (const uint4 *)k,
                                       (const uint4 *)v, bt, seq_lens, B, H, max_blocks, num_pages, ref_blocks,
                                       n_chunks, scale * kLog2e, acc, ml, dev_err);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)(B * H));
    cfg.blockDim = dim3(kD);
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, dense_attn_merge_kernel, seq_lens, B, H, max_blocks, n_chunks,
                              (const float *)acc, (const float *)ml, (__nv_bfloat16 *)out);
}

}  // namespace uocr
