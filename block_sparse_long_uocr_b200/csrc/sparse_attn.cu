// sparse_attn.cu -- exact attention over the selected 16 x 32 tokens.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 step 4:
// attention runs over only the selected blocks (16 blocks x 32 tokens = 512
// tokens per query), never materialising a full score row; section 三: MHA
// with 10 heads of 128 dims.  Per head h of query i at position p:
//   z_t = scale * q . k_t  (t <= p in the selected blocks),
//   out = sum_t softmax(z)_t v_t      (fp32 softmax and accumulation).
//
// Layout of the work: a thread-block cluster of 4 CTAs per (query, head); CTA
// s of the cluster takes selection slots 4s .. 4s+3, one warp per block.
//   * Lane 0 of a warp starts a 1-D bulk copy (TMA, cp.async.bulk + mbarrier)
//     of the block's V tile (8 KiB) into shared memory; the warp streams the K
//     tile (8 KiB) through registers with coalesced 16-byte loads (step t:
//     lane l holds token 2t + l/16, dims 8*(l%16) .. +8), so both reads are in
//     flight together.  A transposed half-warp reduction leaves each lane with
//     one token's score; V is read back from shared memory in the same layout.
//   * The 4 warps' softmax states (m, l, acc[128]) merge in shared memory; the
//     4 CTAs' states merge through distributed shared memory in CTA 0 of the
//     cluster, which writes the bf16 output.  No global scratch, no atomics.
//   * In a decode call the selection comes from block_topk, whose slot layout
//     is known in advance for the 4 local blocks (slots 12..15) and for
//     sequences of at most 16 blocks; those CTAs start their loads before
//     waiting on the top-k kernel (programmatic dependent launch).
// Roofline: HBM-bound, 2 x 8 KiB per (block, head), no reuse across queries.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

constexpr int kAttnWarps = 4;                     // blocks per CTA (one per warp)
constexpr int kAttnCluster = kSel / kAttnWarps;   // CTAs per (query, head)


__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Read a float from the shared memory of CTA `rank` of this cluster at the address of `p`.
__device__ __forceinline__ float ld_dsmem(const float *p, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(p)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Selection slot k of a query with nb causal blocks, as block_topk lays it out,
// when it does not depend on the scores: -2 means "read it from sel".
__device__ __forceinline__ int implicit_slot(int k, int nb) {
    if (nb <= kSel) return k < nb ? k : -1;
    if (k >= kRemote) return nb - kSel + k;
    return -2;
}

__global__ void __launch_bounds__(kAttnWarps * 32)
sparse_attn_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ kc, const uint4 *__restrict__ vc,
                   const int32_t *__restrict__ bt, const int32_t *__restrict__ seq_lens,
                   const int32_t *__restrict__ q_seq, const int32_t *__restrict__ q_pos,
                   const int32_t *__restrict__ sel, int B, int H, int max_blocks, int num_pages,
                   float scale_log2, int implicit_local, int fixed_seq, int head_major, int n_q,
                   __nv_bfloat16 *__restrict__ out, int32_t *dev_err, uint64_t first_wait_ns) {
    __shared__ float s_m[kAttnWarps], s_l[kAttnWarps];
    __shared__ float s_acc[kAttnWarps][kD];
    __shared__ float s_cta_ml[2];
    __shared__ float s_cta_acc[kD];
    __shared__ __align__(8) uint64_t s_bar[kAttnWarps];
    __shared__ __align__(128) uint4 s_v[kAttnWarps][kPageElems / 8];   // one V tile per warp

    const int cl = blockIdx.x / kAttnCluster;
    const int split = (int)cluster_ctarank();    // == blockIdx.x % kAttnCluster
    // head-major order (all queries of head 0 first) keeps one head's K/V hot in L2
    // when many queries share a sequence (prefill); query-major otherwise
    const int h = head_major ? cl / n_q : cl % H;
    const int i = head_major ? cl % n_q : cl / H;
    const int ih = i * H + h;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int slot = split * kAttnWarps + warp;

    float m_w = -INFINITY, l_w = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    // query metadata and (when known in advance) the block are inputs of the call, not
    // outputs of the preceding kernel, so they are read before the dependency wait
    QueryRef r;
    const bool ok = resolve_query(i, seq_lens, q_seq, q_pos, B, max_blocks, dev_err,
                                  threadIdx.x == 0 && split == 0 && h == 0, r, fixed_seq);
    int j = ok && implicit_local ? implicit_slot(slot, r.nb) : -2;
    if (j == -2) {
        pdl_wait();
        j = ok ? __ldg(sel + (size_t)i * kSel + slot) : -1;
    }
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
        const size_t tile = ((size_t)page * H + h) * (kPageElems / 8);
        uint64_t *bar = &s_bar[warp];
        if (lane == 0) {
            mbar_init(bar, 1);
            fence_mbar_init();
            mbar_arrive_expect_tx(bar, kPageElems * 2);
            bulk_copy_g2s(s_v[warp], vc + tile, kPageElems * 2, bar);
        }
        __syncwarp();

        float qf[8];
        bf16x8_to_f32(__ldg(q + ((size_t)i * H + h) * (kD / 8) + (lane & 15)), qf);
        uint4 kv[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) kv[t] = ld_stream(kc + tile + lane + t * 32);
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

        // lane now owns token 2*(lane&15) + lane/16 of the block
        float zt = half_warp_transpose_sum16(z, lane) * scale_log2;
        const int tok = 2 * (lane & 15) + (lane >> 4);
        if (j * kBlock + tok > r.p) zt = -INFINITY;
        m_w = warp_max(zt);                       // finite: token 32j <= p is visible
        const float pt = exp2f(zt - m_w);
        l_w = warp_sum(pt);

        // every lane waits (bounded in wall time) and observes the copy's completion itself
        const bool ready = __all_sync(0xffffffffu, mbar_wait_timed(bar, 0, first_wait_ns, nullptr));
        if (!ready) {
            // The copy did not land in time: report it and drop the block.  Before the warp goes
            // on, a second wait (default limit) lets the copy finish, so that the CTA does not
            // retire with a bulk copy still writing into its shared memory.  If that wait too runs
            // out (a copy stuck for seconds: a broken memory system), the kernel ends regardless,
            // bounded, rather than wait forever.
            if (lane == 0) flag_error(dev_err, UOCR_DEVERR_TIMEOUT);
            mbar_wait_timed(bar, 0, kWaitLimitNs, nullptr);
            m_w = -INFINITY;
            l_w = 0.f;
        } else {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                // weight of token 2t + lane/16, owned by lane (lane & 16) | t
                const float w = __shfl_sync(0xffffffffu, pt, (lane & 16) | t);
                float vf[8];
                bf16x8_to_f32(s_v[warp][t * 32 + lane], vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, vf[e], acc[e]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
        }
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

    // ---- merge the 4 warps; thread d owns output dim d
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
    s_cta_acc[d] = A;
    if (d == 0) {
        s_cta_ml[0] = M;
        s_cta_ml[1] = L;
    }

    // ---- merge the 4 CTAs of the cluster in CTA 0 through distributed shared memory
    cluster_sync();                              // every CTA's state is written and visible
    if (split == 0) {
        float Ms[kAttnCluster], Ls[kAttnCluster], As[kAttnCluster];
        float Mt = -INFINITY;
#pragma unroll
        for (int s = 0; s < kAttnCluster; ++s) {
            Ms[s] = ld_dsmem(&s_cta_ml[0], s);
            Ls[s] = ld_dsmem(&s_cta_ml[1], s);
            As[s] = ld_dsmem(&s_cta_acc[d], s);
            Mt = fmaxf(Mt, Ms[s]);
        }
        float Lt = 0.f, At = 0.f;
        if (Mt != -INFINITY) {
#pragma unroll
            for (int s = 0; s < kAttnCluster; ++s) {
                const float f = exp2f(Ms[s] - Mt);
                Lt = fmaf(Ls[s], f, Lt);
                At = fmaf(As[s], f, At);
            }
        }
        out[(size_t)ih * kD + d] = __float2bfloat16_rn(Lt > 0.f ? At / Lt : 0.f);
    }
    cluster_sync();                              // keep every CTA's shared memory alive until read
    // Warps whose blocks were known in advance never wait on the selection kernel; one thread
    // waits here so that this grid completes after it (its selection output included).
    if (blockIdx.x == 0 && threadIdx.x == 0) pdl_wait();
}

cudaError_t launch_sparse_attn(const LaunchCtx &c, const void *q, const void *k, const void *v,
                               const int32_t *bt, const int32_t *seq_lens, const int32_t *q_seq,
                               const int32_t *q_pos, const int32_t *sel, int n_q, int B, int H,
                               int max_blocks, int num_pages, float scale, void *out,
                               bool implicit_local, int fixed_seq, bool head_major, int32_t *dev_err) {
    const long long grid = (long long)n_q * H * kAttnCluster;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kAttnCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kAttnWarps * 32);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, sparse_attn_kernel, (const uint4 *)q, (const uint4 *)k, (const uint4 *)v, bt,
                              seq_lens, q_seq, q_pos, sel, B, H, max_blocks, num_pages, scale * kLog2e,
                              implicit_local ? 1 : 0, fixed_seq, head_major ? 1 : 0, n_q, (__nv_bfloat16 *)out,
                              dev_err, c.first_wait_ns);
}

}  // namespace uocr
