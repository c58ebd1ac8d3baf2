// rope_append.cu -- page2d rotary embedding of a decode step's new tokens and the
// append of their keys / values to the paged caches (the step before the scan).
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 四 (page2d):
// the 64 frequency pairs of a 128-dim head are split between two axes -- one
// pair for the page coordinate (page % 2), the other 63 for the in-page token
// offset, resampled over the whole spectrum -- and the angles are laid out as
// cos/sin of cat(ang, ang) (rotate-half: pair i = dims i and i + 64).  Section
// 六: token axis theta = 10000, page axis theta = 256.  The main attention and
// the indexer share the same coordinates; the cache stores rotated keys.
//
// One CTA per new token: the 64 angles are formed in fp64 (token offsets reach
// 1e5 radians, where an fp32 product alone would be off by ~0.01 rad), reduced
// to [-pi, pi] and passed to sincosf; then the H query heads and the indexer
// query are rotated in place, and the H key heads, the indexer key (rotated) and
// the H value heads (unchanged) are written to the token's cache row, 16 bytes
// (8 pairs) per thread and step.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

namespace {
constexpr int kPairs = kD / 2;     // 64
constexpr int kRopeThreads = 128;
}  // namespace

__global__ void __launch_bounds__(kRopeThreads)
rope_append_kernel(__nv_bfloat16 *__restrict__ q, __nv_bfloat16 *__restrict__ idx_q,
                   const __nv_bfloat16 *__restrict__ k_new, const __nv_bfloat16 *__restrict__ v_new,
                   const __nv_bfloat16 *__restrict__ idx_k_new, const int32_t *__restrict__ tok_pos,
                   const int32_t *__restrict__ page_pos, const int32_t *__restrict__ q_seq,
                   const int32_t *__restrict__ q_pos, const int32_t *__restrict__ bt,
                   const int32_t *__restrict__ seq_lens, int B, int H, int max_blocks, int num_pages,
                   __nv_bfloat16 *__restrict__ k_cache, __nv_bfloat16 *__restrict__ v_cache,
                   __nv_bfloat16 *__restrict__ idx_k_cache, RopeFreqs freqs, int32_t *dev_err) {
    __shared__ float s_cos[kPairs], s_sin[kPairs];
    const int i = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_wait();

    if (tid < kPairs) {
        const int page_mod2 = ((__ldg(page_pos + i) % 2) + 2) % 2;
        const double coord = tid < kPairs - UOCR_ROPE_PAGE_PAIRS ? (double)__ldg(tok_pos + i) : (double)page_mod2;
        double a = coord * freqs.inv[tid];
        const double two_pi = 6.283185307179586476925;
        a -= two_pi * rint(a / two_pi);
        float sn, cs;
        sincosf((float)a, &sn, &cs);
        s_cos[tid] = cs;
        s_sin[tid] = sn;
    }
    __syncthreads();

    QueryRef r;
    const bool ok = resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err, tid == 0, r);
    int page = -1;
    int row = 0;
    if (ok && r.p >= 0) {
        page = __ldg(bt + (size_t)r.b * max_blocks + r.p / kBlock);
        row = r.p % kBlock;
        if ((unsigned)page >= (unsigned)num_pages) {
            if (tid == 0) flag_error(dev_err, UOCR_DEVERR_PAGE);
            page = -1;
        }
    }

    // rotation work items: (vector v, chunk c) for v in [q heads..., idx_q, k heads..., idx_k]; chunk c
    // holds pairs 8c .. 8c + 7, i.e. dims 8c .. 8c + 7 and 64 + 8c .. 64 + 8c + 7 (two 16-byte loads)
    const int n_vec = 2 * H + 2;
    for (int w = tid; w < n_vec * (kPairs / 8); w += kRopeThreads) {
        const int v = w / (kPairs / 8), c = w % (kPairs / 8);
        const __nv_bfloat16 *src;
        __nv_bfloat16 *dst;
        if (v < H) {
            src = dst = q + ((size_t)i * H + v) * kD;
        } else if (v == H) {
            src = dst = idx_q + (size_t)i * kDIdx;
        } else if (v < 2 * H + 1) {
            const int h = v - H - 1;
            src = k_new + ((size_t)i * H + h) * kD;
            dst = page >= 0 ? k_cache + (((size_t)page * H + h) * kBlock + row) * kD : nullptr;
        } else {
            src = idx_k_new + (size_t)i * kDIdx;
            dst = page >= 0 ? idx_k_cache + ((size_t)page * kBlock + row) * kDIdx : nullptr;
        }
        if (!dst) continue;
        const uint4 lo = reinterpret_cast<const uint4 *>(src)[c];
        const uint4 hi = reinterpret_cast<const uint4 *>(src + kPairs)[c];
        const __nv_bfloat162 *l2 = reinterpret_cast<const __nv_bfloat162 *>(&lo);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&hi);
        uint4 olo, ohi;
        __nv_bfloat162 *ol = reinterpret_cast<__nv_bfloat162 *>(&olo);
        __nv_bfloat162 *oh = reinterpret_cast<__nv_bfloat162 *>(&ohi);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x0 = __bfloat1622float2(l2[e]), x1 = __bfloat1622float2(h2[e]);
            const int d = 8 * c + 2 * e;
            const float c0 = s_cos[d], s0 = s_sin[d], c1 = s_cos[d + 1], s1 = s_sin[d + 1];
            ol[e] = __floats2bfloat162_rn(x0.x * c0 - x1.x * s0, x0.y * c1 - x1.y * s1);
            oh[e] = __floats2bfloat162_rn(x1.x * c0 + x0.x * s0, x1.y * c1 + x0.y * s1);
        }
        reinterpret_cast<uint4 *>(dst)[c] = olo;
        reinterpret_cast<uint4 *>(dst + kPairs)[c] = ohi;
    }
    // values are cached as they are
    if (page >= 0) {
        for (int w = tid; w < H * (kD / 8); w += kRopeThreads) {
            const int h = w / (kD / 8), c = w % (kD / 8);
            const uint4 val = __ldg(reinterpret_cast<const uint4 *>(v_new + ((size_t)i * H + h) * kD) + c);
            reinterpret_cast<uint4 *>(v_cache + (((size_t)page * H + h) * kBlock + row) * kD)[c] = val;
        }
    }
}

RopeFreqs rope_freqs() {
    RopeFreqs f;
    const int n_tok = kPairs - UOCR_ROPE_PAGE_PAIRS;
    for (int i = 0; i < kPairs; ++i) {
        if (i < n_tok)
            f.inv[i] = pow((double)UOCR_ROPE_THETA_TOKEN, -(double)i / (double)n_tok);
        else
            f.inv[i] = pow((double)UOCR_ROPE_THETA_PAGE, -(double)(i - n_tok) / (double)UOCR_ROPE_PAGE_PAIRS);
    }
    return f;
}

cudaError_t launch_rope_append(const LaunchCtx &c, void *q, void *idx_q, const void *k_new, const void *v_new,
                               const void *idx_k_new, const int32_t *tok_pos, const int32_t *page_pos,
                               const int32_t *q_seq, const int32_t *q_pos, const int32_t *bt,
                               const int32_t *seq_lens, int n, int B, int H, int max_blocks, int num_pages,
                               void *k_cache, void *v_cache, void *idx_k_cache, int32_t *dev_err) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n);
    cfg.blockDim = dim3(kRopeThreads);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, rope_append_kernel, (__nv_bfloat16 *)q, (__nv_bfloat16 *)idx_q,
                              (const __nv_bfloat16 *)k_new, (const __nv_bfloat16 *)v_new,
                              (const __nv_bfloat16 *)idx_k_new, tok_pos, page_pos, q_seq, q_pos, bt, seq_lens, B,
                              H, max_blocks, num_pages, (__nv_bfloat16 *)k_cache, (__nv_bfloat16 *)v_cache,
                              (__nv_bfloat16 *)idx_k_cache, rope_freqs(), dev_err);
}

}  // namespace uocr
