// prefill_attn.cu -- block-centric sparse attention for a prefill chunk.
//
// Same arithmetic as sparse_attn.cu (Unlimited-OCR-2 walk-through,
// news.rkmt.cn/news/25027, section 五 step 4: exact softmax attention of each
// query over its 16 selected 32-token blocks), organised for many queries of
// one sequence.  Query-by-query gathering would read every selected (block,
// head) tile once per query that picked it -- ~16 times per tile on average in
// a 2048-query chunk, and ~130 times for the local-window blocks that 32
// consecutive queries share.  Instead:
//   1. invert the selection: per logical block, the list of (query, slot)
//      entries that selected it (count with atomics, one-CTA exclusive scan,
//      fill);
//   2. one CTA per (block, head) copies the block's K and V tiles (2 x 8 KiB)
//      into shared memory with 1-D bulk copies (TMA) and runs every entry of
//      its list against them, one warp per entry, writing the entry's partial
//      softmax state (m, l, acc[128]) to the workspace.  Blocks are visited
//      from the last one down, so the heavily shared local-window blocks start
//      first;
//   3. one CTA per (query, head) merges its 16 partials (flash-decoding) and
//      writes the bf16 output.
// Each (block, head) tile is read from memory once per chunk.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

namespace {
constexpr int kInvThreads = 256;
constexpr int kScanThreads = 1024;
constexpr int kBAWarps = 4;
}  // namespace

__global__ void __launch_bounds__(kInvThreads)
prefill_count_kernel(const int32_t *__restrict__ sel, int n_entries, int max_blocks, int32_t *counts) {
    pdl_wait();
    const int e = blockIdx.x * kInvThreads + threadIdx.x;
    if (e < n_entries) {
        const int j = sel[e];
        if (j >= 0 && j < max_blocks) atomicAdd(counts + j, 1);
    }
}

// One CTA: offsets = exclusive prefix sum of counts; cursor = offsets.
__global__ void __launch_bounds__(kScanThreads)
prefill_scan_kernel(const int32_t *__restrict__ counts, int max_blocks, int32_t *__restrict__ offsets,
                    int32_t *__restrict__ cursor) {
    __shared__ int warp_tot[kScanThreads / 32];
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (max_blocks + kScanThreads - 1) / kScanThreads;
    const int lo = tid * per, hi = min(max_blocks, lo + per);
    int mine = 0;
    for (int j = lo; j < hi; ++j) mine += counts[j];
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        warp_tot[lane] = wi - w;
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - mine;
    for (int j = lo; j < hi; ++j) {
        offsets[j] = run;
        cursor[j] = run;
        run += counts[j];
    }
}

__global__ void __launch_bounds__(kInvThreads)
prefill_fill_kernel(const int32_t *__restrict__ sel, int n_entries, int max_blocks, int32_t *cursor,
                    int32_t *__restrict__ list) {
    pdl_wait();
    const int e = blockIdx.x * kInvThreads + threadIdx.x;
    if (e < n_entries) {
        const int j = sel[e];
        if (j >= 0 && j < max_blocks) list[atomicAdd(cursor + j, 1)] = e;
    }
}

__global__ void __launch_bounds__(kBAWarps * 32)
prefill_block_attn_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ kc, const uint4 *__restrict__ vc,
                          const int32_t *__restrict__ bt_row, const int32_t *__restrict__ q_pos,
                          const int32_t *__restrict__ counts, const int32_t *__restrict__ offsets,
                          const int32_t *__restrict__ list, int H, int max_blocks, int num_pages, float scale_log2,
                          float *__restrict__ part_acc, float *__restrict__ part_ml, int32_t *dev_err) {
    __shared__ __align__(128) uint4 s_k[kPageElems / 8];
    __shared__ __align__(128) uint4 s_v[kPageElems / 8];
    __shared__ __align__(8) uint64_t s_bar;

    const int j = max_blocks - 1 - (int)(blockIdx.x / H);
    const int h = (int)(blockIdx.x % H);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_wait();
    const int n = counts[j];
    if (n == 0) return;
    const int off = offsets[j];
    const int page = __ldg(bt_row + j);
    bool have = (unsigned)page < (unsigned)num_pages;
    if (!have && threadIdx.x == 0) flag_error(dev_err, UOCR_DEVERR_PAGE);

    if (have) {
        if (threadIdx.x == 0) {
            const size_t tile = ((size_t)page * H + h) * (kPageElems / 8);
            mbar_init(&s_bar, 1);
            fence_mbar_init();
            mbar_arrive_expect_tx(&s_bar, 2 * kPageElems * 2);
            bulk_copy_g2s(s_k, kc + tile, kPageElems * 2, &s_bar);
            bulk_copy_g2s(s_v, vc + tile, kPageElems * 2, &s_bar);
        }
        __syncthreads();
        if (!mbar_wait_timed(&s_bar, 0, 2000000000ull, nullptr)) {
            if (threadIdx.x == 0) flag_error(dev_err, UOCR_DEVERR_TIMEOUT);
            mbar_wait_timed(&s_bar, 0, 2000000000ull, nullptr);
            have = false;
        }
    }

    const int tok = 2 * (lane & 15) + (lane >> 4);
    for (int e = warp; e < n; e += kBAWarps) {
        const int entry = __ldg(list + off + e);
        const int i = entry >> 4;
        const size_t slot = ((size_t)i * H + h) * kSel + (entry & 15);
        float m_w = -INFINITY, l_w = 0.f;
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
        if (have) {
            const int p = __ldg(q_pos + i);
            float qf[8];
            bf16x8_to_f32(__ldg(q + ((size_t)i * H + h) * (kD / 8) + (lane & 15)), qf);
            float z[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                float kf[8];
                bf16x8_to_f32(s_k[t * 32 + lane], kf);
                float a = qf[0] * kf[0];
#pragma unroll
                for (int c = 1; c < 8; ++c) a = fmaf(qf[c], kf[c], a);
                z[t] = a;
            }
            float zt = half_warp_transpose_sum16(z, lane) * scale_log2;
            if (j * kBlock + tok > p) zt = -INFINITY;
            m_w = warp_max(zt);                   // finite: a selected block has token 32j <= p
            const float pt = exp2f(zt - m_w);
            l_w = warp_sum(pt);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float w = __shfl_sync(0xffffffffu, pt, (lane & 16) | t);
                float vf[8];
                bf16x8_to_f32(s_v[t * 32 + lane], vf);
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = fmaf(w, vf[c], acc[c]);
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 16);
        }
        if (lane < 16) {
            float4 *dst = reinterpret_cast<float4 *>(part_acc + slot * kD + lane * 8);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        if (lane == 0) {
            part_ml[slot * 2] = m_w;
            part_ml[slot * 2 + 1] = l_w;
        }
    }
}

// One CTA per (query, head); thread d owns output dim d.
__global__ void __launch_bounds__(kD)
prefill_merge_kernel(const int32_t *__restrict__ sel, const float *__restrict__ part_acc,
                     const float *__restrict__ part_ml, int H, __nv_bfloat16 *__restrict__ out) {
    const int ih = blockIdx.x;
    const int i = ih / H;
    const int d = threadIdx.x;
    pdl_wait();
    float M = -INFINITY;
    int valid = 0;
#pragma unroll
    for (int k = 0; k < kSel; ++k) {
        if (__ldg(sel + (size_t)i * kSel + k) >= 0) {
            valid |= 1 << k;
            M = fmaxf(M, part_ml[((size_t)ih * kSel + k) * 2]);
        }
    }
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int k = 0; k < kSel; ++k) {
            if (!(valid >> k & 1)) continue;
            const size_t slot = (size_t)ih * kSel + k;
            const float f = exp2f(part_ml[slot * 2] - M);
            L = fmaf(part_ml[slot * 2 + 1], f, L);
            A = fmaf(part_acc[slot * kD + d], f, A);
        }
    }
    out[(size_t)ih * kD + d] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
}

// ------------------------------------------------------------------ host side
size_t prefill_attn_workspace(int n_q, int H, int max_blocks, PrefillAttnWs *w) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    size_t off = 0;
    PrefillAttnWs l{};
    l.counts_off = off;
    off += up((size_t)max_blocks * 4);
    l.offsets_off = off;
    off += up((size_t)max_blocks * 4);
    l.cursor_off = off;
    off += up((size_t)max_blocks * 4);
    l.list_off = off;
    off += up((size_t)n_q * kSel * 4);
    l.ml_off = off;
    off += up((size_t)n_q * H * kSel * 2 * 4);
    l.acc_off = off;
    off += up((size_t)n_q * H * kSel * kD * 4);
    if (w) *w = l;
    return off;
}

cudaError_t launch_prefill_attn(const LaunchCtx &c, const void *q, const void *k, const void *v,
                                const int32_t *bt_row, const int32_t *q_pos, const int32_t *sel, int n_q, int H,
                                int max_blocks, int num_pages, float scale, void *out, void *ws,
                                int32_t *dev_err) {
    PrefillAttnWs w;
    prefill_attn_workspace(n_q, H, max_blocks, &w);
    char *base = (char *)ws;
    int32_t *counts = (int32_t *)(base + w.counts_off);
    int32_t *offsets = (int32_t *)(base + w.offsets_off);
    int32_t *cursor = (int32_t *)(base + w.cursor_off);
    int32_t *list = (int32_t *)(base + w.list_off);
    float *ml = (float *)(base + w.ml_off);
    float *acc = (float *)(base + w.acc_off);
    const int n_entries = n_q * kSel;

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // every kernel here follows another kernel of the same call

    cfg.gridDim = dim3((unsigned)((n_entries + kInvThreads - 1) / kInvThreads));
    cfg.blockDim = dim3(kInvThreads);
    cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_count_kernel, sel, n_entries, max_blocks, counts);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kScanThreads);
    e = cudaLaunchKernelEx(&cfg, prefill_scan_kernel, (const int32_t *)counts, max_blocks, offsets, cursor);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)((n_entries + kInvThreads - 1) / kInvThreads));
    cfg.blockDim = dim3(kInvThreads);
    e = cudaLaunchKernelEx(&cfg, prefill_fill_kernel, sel, n_entries, max_blocks, cursor, list);
    if (e != cudaSuccess) return e;
    const long long ctas = (long long)max_blocks * H;
    if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(kBAWarps * 32);
    e = cudaLaunchKernelEx(&cfg, prefill_block_attn_kernel, (const uint4 *)q, (const uint4 *)k, (const uint4 *)v,
                           bt_row, q_pos, (const int32_t *)counts, (const int32_t *)offsets, (const int32_t *)list,
                           H, max_blocks, num_pages, scale * kLog2e, acc, ml, dev_err);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)(n_q * H));
    cfg.blockDim = dim3(kD);
    return cudaLaunchKernelEx(&cfg, prefill_merge_kernel, sel, (const float *)acc, (const float *)ml, H,
                              (__nv_bfloat16 *)out);
}

}  // namespace uocr
