// prefill_attn.cu -- block-centric sparse attention for a prefill chunk: the
// entries that the local-window kernel (prefill_local.cu) does not take.
//
// Same arithmetic as sparse_attn.cu (Unlimited-OCR-2 walk-through,
// news.rkmt.cn/news/25027, section 五 step 4: exact softmax attention of each
// query over its selected 32-token blocks), organised for many queries of one
// sequence.  Query-by-query gathering would read every selected (block, head)
// tile once per query that picked it -- ~12 times per remote tile on average in
// a 2048-query chunk.  Instead:
//   1. the selection is classified per 128-query tile (prefill_local.cu): the
//      local-window entries of tiles whose windows fit one 8-block window go
//      to the tensor-core local kernel, which runs on a quarter of the SMs
//      beside step 3; every other entry (the 12 remote blocks of a query, and
//      all entries of other tiles) stays here, counted per block;
//   2. the inversion: per logical block, the list of (query, slot) entries
//      that selected it (one kernel places the lists by the prefix sums of the
//      counts, writes them and cuts them into items of 16 entries);
//   3. one warp per (item, head) unit computes the item's 16 x 32 score
//      tile S = Q K^T and, after a register-resident fp32 softmax per row, the
//      16 x 128 tile P V on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
//      accumulate), writing each entry's partial state: the row maximum m and
//      the weight sum l in fp32, and the unnormalised output acc = sum_t
//      2^(z_t - m) v_t in bf16 (the partial output in the output dtype, the
//      softmax statistics in fp32; |acc| <= l max|v|, so its rounding adds at
//      most 2^-9 max|v| to the result after the merge divides by the summed
//      weights, the size of the output's own bf16 rounding, and halves the
//      partials' traffic);
//   4. the merge kernel (prefill_local.cu) combines each (query, head)'s
//      partials, its local window's included: out = sum_k 2^(m_k - M) acc_k /
//      sum_k 2^(m_k - M) l_k.
// Each (block, head) tile is read from memory about once per chunk (an item after
// the first of the same tile runs beside it and finds it in L2).
//
// Tensor-core layout of step 3.  The contraction index of S = Q K^T is the head
// dimension, and any permutation of it applied to both operands leaves S
// unchanged; this kernel assigns lane (r, t) = (lane / 4, lane % 4) the dims
// 32u + 8t .. 32u + 8t + 7 for the k-steps 2u and 2u + 1, so that every A (query)
// and B (key) fragment is one 16-byte load of a row: no shuffles for S.  P V
// needs V transposed: the warp copies its V tile into shared memory with
// cp.async, 16-byte chunk c of token x at chunk position c ^ (x & 7), and
// ldmatrix.trans reads it without bank conflicts.  P is rounded to bf16 for the
// tensor cores and the row sum l is taken over the rounded weights, so the
// output is an exact convex combination of the values (the normalised weights
// move by at most ~2^-8 of their size, the output by ~2^-9 times the range of
// the values).  An item holds at most 16 entries -- a remote block is chosen by
// ~12 queries of a chunk on average -- below the 64-row minimum tile of
// tcgen05, so these products stay on the warp-level tensor-core instructions.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace uocr {

namespace {
constexpr int kInvThreads = 256;
constexpr int kInvPerThread = 8;
constexpr int kInvTile = kInvThreads * kInvPerThread;   // blocks per prefix-sum tile of the inversion
constexpr int kInvEntries = 4;   // selection entries per thread of the inversion (each CTA recomputes
                                 // the prefix sums, so fewer CTAs re-read fewer counts)
constexpr int kItemRows = 16;
constexpr int kMmaWarps = 2;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// L2 eviction policies (PTX createpolicy): the K/V tiles stream through L2 once per chunk and go
// first; the partials, which the merge kernel of the same call reads back, stay.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void st_u32_pol(uint32_t *p, uint32_t v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(p), "r"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_f2_pol(float *p, float a, float b, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(a), "f"(b), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async16_pol(uint32_t dst, const void *src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&d)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(addr)
                 : "memory");
}

// d += A (16 x 16, row) * B (16 x 8, col); bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 pair (lo in the low half) and the sum of the two rounded values.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi, float &sum) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    sum += __low2float(v) + __high2float(v);
    return *reinterpret_cast<const uint32_t *>(&v);
}
}  // namespace

// The selection inverted in one grid: CTA b places the entries e in [1024 b, 1024 b + 1024) in the
// per-block lists, grouped by block ({entry = query * 16 + slot, position of the query}), and
// writes the work items of the blocks j with j % gridDim.x == b: block j with n_j entries gives
// items (j, 0) .. (j, ceil(n_j / 16) - 1), in block order, each recorded as {j, page of j, first
// entry, entries (<= 16)} so that a warp needs one load.  Each CTA computes the exclusive prefix
// sums of counts (each block's first list position and first item) itself, 2048 blocks at a time
// (8 KiB of counts from L2 per tile); a block's entries take consecutive list positions from a
// counter per block (fill, zero before the call).
__global__ void __launch_bounds__(kInvThreads)
prefill_invert_kernel(const int32_t *counts, const int32_t *__restrict__ bt_row, const int32_t *sel,
                      const int32_t *__restrict__ q_pos, int n_entries, int max_blocks, int32_t *fill,
                      int4 *__restrict__ items, int32_t *__restrict__ n_items, int2 *__restrict__ list) {
    __shared__ int s_c[kInvTile], s_g[kInvTile];   // exclusive prefixes (entries, items) inside the tile
    __shared__ int s_wc[kInvThreads / 32], s_wg[kInvThreads / 32];
    // The counts and the classified selection come from the classification, the preceding kernel.
    // Once every CTA is past that wait, the local-window kernel may start; it waits for this grid
    // before anything else.
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // this thread's entries (kInvEntries, kInvThreads apart), loaded before the scan so that the
    // loads overlap it
    int ej[kInvEntries], ep[kInvEntries];
#pragma unroll
    for (int k = 0; k < kInvEntries; ++k) {
        const int e = (blockIdx.x * kInvEntries + k) * kInvThreads + tid;
        ej[k] = -1;
        ep[k] = 0;
        if (e < n_entries) {   // both loads in flight together
            ej[k] = __ldcg(sel + e);
            ep[k] = __ldg(q_pos + e / kSel);
            if (ej[k] >= max_blocks) ej[k] = -1;
        }
    }
    int base_c = 0, base_g = 0;   // entries and items of the blocks before the tile
    const int G = (int)gridDim.x;
    for (int t0 = 0; t0 < max_blocks; t0 += kInvTile) {
        // the first block of the tile whose items this thread records (local index x with
        // (t0 + x) % G == blockIdx.x), and its page, loaded ahead of the prefix sums
        const int len = min(kInvTile, max_blocks - t0);
        const int first = (int)((blockIdx.x + (unsigned)G - (unsigned)(t0 % G)) % (unsigned)G);
        const int x0 = first + tid * G;
        const int page0 = x0 < len ? __ldg(bt_row + t0 + x0) : 0;
        // thread tid sums blocks t0 + 8 tid .. t0 + 8 tid + 7
        int c[kInvPerThread], sc = 0, sg = 0;
#pragma unroll
        for (int k = 0; k < kInvPerThread; ++k) {
            const int jb = t0 + kInvPerThread * tid + k;
            c[k] = jb < max_blocks ? __ldcg(counts + jb) : 0;
            sc += c[k];
            sg += (c[k] + kItemRows - 1) / kItemRows;
        }
        int ic = sc, ig = sg;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nc = __shfl_up_sync(0xffffffffu, ic, o);
            const int ng = __shfl_up_sync(0xffffffffu, ig, o);
            if (lane >= o) {
                ic += nc;
                ig += ng;
            }
        }
        if (lane == 31) {
            s_wc[warp] = ic;
            s_wg[warp] = ig;
        }
        __syncthreads();
        int rc = ic - sc, rg = ig - sg, tot_c = 0, tot_g = 0;
#pragma unroll
        for (int w = 0; w < kInvThreads / 32; ++w) {
            if (w < warp) {
                rc += s_wc[w];
                rg += s_wg[w];
            }
            tot_c += s_wc[w];
            tot_g += s_wg[w];
        }
#pragma unroll
        for (int k = 0; k < kInvPerThread; ++k) {
            s_c[kInvPerThread * tid + k] = rc;
            s_g[kInvPerThread * tid + k] = rg;
            rc += c[k];
            rg += (c[k] + kItemRows - 1) / kItemRows;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kInvEntries; ++k) {
            const int j = ej[k];
            if (j >= t0 && j < t0 + kInvTile)
                list[base_c + s_c[j - t0] + atomicAdd(fill + j, 1)] =
                    make_int2((blockIdx.x * kInvEntries + k) * kInvThreads + tid, ep[k]);
        }
        // the items of this CTA's blocks in the tile
        for (int x = x0; x < len; x += kInvThreads * G) {
            const int cnt = (x + 1 < kInvTile ? s_c[x + 1] : tot_c) - s_c[x];
            if (cnt == 0) continue;
            const int jb = t0 + x;
            const int page = x == x0 ? page0 : __ldg(bt_row + jb);
            const int g0 = base_g + s_g[x], c0 = base_c + s_c[x];
            for (int k = 0; k * kItemRows < cnt; ++k)
                items[g0 + k] = make_int4(jb, page, c0 + k * kItemRows, min(kItemRows, cnt - k * kItemRows));
        }
        base_c += tot_c;
        base_g += tot_g;
        __syncthreads();   // the next tile reuses s_c, s_g, s_wc, s_wg
    }
    if (blockIdx.x == 0 && tid == 0) *n_items = base_g;
}

// One unit of work: (item, head) and the item's record and entries.
struct Unit {
    int w;          // unit index, or -1 past the end
    int j, page, rows, h;
    int2 ea, eb;    // entries {query * 16 + slot, position} of rows r and r + 8
};

__device__ __forceinline__ Unit load_unit(int w, int n_work, int H, const int4 *items, const int2 *list, int r) {
    Unit u;
    u.w = w < n_work ? w : -1;
    if (u.w < 0) {
        u.j = u.page = u.h = 0;
        u.rows = 1;
        u.ea = u.eb = make_int2(0, 0);
        return u;
    }
    // written by the inversion earlier in the same call, read through L2
    const int4 rec = __ldcg(items + w / H);
    u.j = rec.x;
    u.page = rec.y;
    u.rows = rec.w;
    u.h = w % H;
    // rows past the item's end repeat its last entry and store nothing
    u.ea = __ldcg(list + rec.z + min(r, rec.w - 1));
    u.eb = __ldcg(list + rec.z + min(r + 8, rec.w - 1));
    return u;
}

// Per-warp staging: 16-byte chunk c of row x of K and Q at chunk c ^ ((x & 1) << 2) (the
// fragment reads touch two rows per 8-lane phase), of V at c ^ (x & 7) (ldmatrix.trans reads
// eight consecutive rows of one chunk).
struct WarpStage {
    uint4 k[kBlock * kD / 8];
    uint4 v[kBlock * kD / 8];
    uint4 q[kItemRows * kD / 8];
};

// Persistent: each warp takes its units, unit = (item, head), in order from a counter (sched,
// zero before the call), one unit ahead of the one it computes; heads are innermost so that the
// items of one block run side by side.  The counter lets the CTAs that start late (beside the
// local-window kernel, which holds most of a few SMs' shared memory) take fewer units.  Each warp
// pipelines its units: the next unit's Q and K copies start once this unit's scores are computed,
// its V copy once this unit's P V is done, so every copy overlaps the math of the unit before it
// (cp.async groups, waited for with wait_group 1).
//
// Launched after the local-window kernel, whose CTAs let this grid start once they are past their
// own wait for the inversion: the lists and items are complete here (read through L2), and this
// grid does not wait for the local kernel before its work.  One thread waits for it at the end, so
// that this grid completes only after the local kernel and the merge, which waits for this grid,
// reads both kernels' partials.
__global__ void __launch_bounds__(kMmaWarps * 32)
prefill_block_mma_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ kc, const uint4 *__restrict__ vc,
                         const int2 *__restrict__ list, const int4 *__restrict__ items,
                         const int32_t *__restrict__ n_items, int32_t *sched, int H, int num_pages,
                         float scale_log2, __nv_bfloat16 *__restrict__ part_o, float *__restrict__ part_ml,
                         int32_t *dev_err) {
    __shared__ __align__(128) WarpStage stage[kMmaWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, t = lane & 3;
    const uint32_t sk = smem_addr(stage[warp].k), sv = smem_addr(stage[warp].v), sq = smem_addr(stage[warp].q);
    const uint4 *k_s = stage[warp].k, *q_s = stage[warp].q;

    const uint64_t pol_kv = l2_evict_first(), pol_part = l2_evict_last();
    // the merge kernel may start its prologue; it waits for this grid before reading the partials
    pdl_launch_dependents();
    const int n_work = __ldcg(n_items) * H;
    auto take = [&]() {
        int w = 0;
        if (lane == 0) w = atomicAdd(sched, 1);
        return __shfl_sync(0xffffffffu, w, 0);
    };

    auto page_ok = [&](const Unit &u) { return (unsigned)u.page < (unsigned)num_pages; };
    // Q rows (16) and the K tile of unit u; then its V tile
    auto issue_qk = [&](const Unit &u) {
        if (u.w >= 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int x = k * 32 + lane, row = x >> 4, c = x & 15;
                const int src = (row & 7) * 4;
                const int ea = __shfl_sync(0xffffffffu, u.ea.x, src), eb = __shfl_sync(0xffffffffu, u.eb.x, src);
                const int ent = row < 8 ? ea : eb;
                // rows past the item's end are not copied: their scores and outputs are computed
                // from whatever the buffer holds and never stored (each row of an MMA's result
                // depends on its own row of A alone)
                if (row < u.rows)
                    cp_async16(sq + (uint32_t)((row * 16 + (c ^ ((row & 1) << 2))) * 16),
                               q + ((size_t)(ent >> 4) * H + u.h) * (kD / 8) + c);
            }
            if (page_ok(u)) {
                const uint4 *src = kc + ((size_t)u.page * H + u.h) * (kPageElems / 8);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int x = k * 32 + lane, tok = x >> 4, c = x & 15;
                    cp_async16_pol(sk + (uint32_t)((tok * 16 + (c ^ ((tok & 1) << 2))) * 16), src + x, pol_kv);
                }
            }
        }
        cp_async_commit();
    };
    auto issue_v = [&](const Unit &u) {
        if (u.w >= 0 && page_ok(u)) {
            const uint4 *src = vc + ((size_t)u.page * H + u.h) * (kPageElems / 8);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int x = k * 32 + lane, tok = x >> 4, c = x & 15;
                cp_async16_pol(sv + (uint32_t)((tok * 16 + (c ^ (tok & 7))) * 16), src + x, pol_kv);
            }
        }
        cp_async_commit();
    };

    Unit cur = load_unit(take(), n_work, H, items, list, r);
    Unit nxt = cur;
    if (cur.w >= 0) {
        issue_qk(cur);
        issue_v(cur);
        nxt = load_unit(take(), n_work, H, items, list, r);
    }

    while (cur.w >= 0) {
        // ---- S = Q K^T (rows r, r + 8; tokens 8 nt + 2t, 8 nt + 2t + 1) from this unit's Q, K
        cp_async_wait_1();
        __syncwarp();
        float s[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        const int sw = (r & 1) << 2;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 qa = q_s[r * 16 + ((4 * u + t) ^ sw)];
            const uint4 qb = q_s[(r + 8) * 16 + ((4 * u + t) ^ sw)];
            uint4 kf[4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) kf[nt] = k_s[(8 * nt + r) * 16 + ((4 * u + t) ^ sw)];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                mma_bf16(s[nt], qa.x, qb.x, qa.y, qb.y, kf[nt].x, kf[nt].y);
                mma_bf16(s[nt], qa.z, qb.z, qa.w, qb.w, kf[nt].z, kf[nt].w);
            }
        }
        __syncwarp();       // Q and K read: the next unit's copies may land
        issue_qk(nxt);

        // ---- causal mask t <= p, scale, row maxima and sums over the quad
        const int pa = cur.ea.y, pb = cur.eb.y;
        const int t0 = cur.j * kBlock + 2 * t;
        float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
        // a block wholly at or before every row's position (every remote block) needs no mask
        const bool visible = cur.j * kBlock + kBlock - 1 <= __reduce_min_sync(0xffffffffu, min(pa, pb));
        if (visible) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    s[nt][e] *= scale_log2;
                    s[nt][2 + e] *= scale_log2;
                    ma = fmaxf(ma, s[nt][e]);
                    mb = fmaxf(mb, s[nt][2 + e]);
                }
        } else {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = t0 + 8 * nt + e;
                    s[nt][e] = tok <= pa ? s[nt][e] * scale_log2 : -INFINITY;
                    s[nt][2 + e] = tok <= pb ? s[nt][2 + e] * scale_log2 : -INFINITY;
                    ma = fmaxf(ma, s[nt][e]);
                    mb = fmaxf(mb, s[nt][2 + e]);
                }
        }
#pragma unroll
        for (int x = 1; x < 4; x <<= 1) {
            ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, x));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, x));
        }
        // finite: a selected block holds a token at or before the query
        uint32_t pf[4][2];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            pf[nt][0] = pack_bf16(exp2f(s[nt][0] - ma), exp2f(s[nt][1] - ma), la);
            pf[nt][1] = pack_bf16(exp2f(s[nt][2] - mb), exp2f(s[nt][3] - mb), lb);
        }
#pragma unroll
        for (int x = 1; x < 4; x <<= 1) {
            la += __shfl_xor_sync(0xffffffffu, la, x);
            lb += __shfl_xor_sync(0xffffffffu, lb, x);
        }

        // ---- O = P V: k-steps of 16 tokens, n-tiles of 8 dims, V^T fragments by ldmatrix.trans
        cp_async_wait_1();
        __syncwarp();
        float o[16][4];
#pragma unroll
        for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int tok = 16 * kk + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                const int c = 2 * np + (lane >> 4);
                uint32_t b[4];
                ldsm_x4_trans(b, sv + (uint32_t)((tok * 16 + (c ^ (tok & 7))) * 16));
                mma_bf16(o[2 * np], pf[2 * kk][0], pf[2 * kk][1], pf[2 * kk + 1][0], pf[2 * kk + 1][1], b[0], b[1]);
                mma_bf16(o[2 * np + 1], pf[2 * kk][0], pf[2 * kk][1], pf[2 * kk + 1][0], pf[2 * kk + 1][1], b[2],
                         b[3]);
            }
        }
        __syncwarp();       // V read: the next unit's V may land
        issue_v(nxt);

        if (!page_ok(cur)) {
            // no tile was copied: the entries get an empty partial
            if (lane == 0) flag_error(dev_err, UOCR_DEVERR_PAGE);
            ma = mb = -INFINITY;
            la = lb = 0.f;
#pragma unroll
            for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        }
        const int ia = cur.ea.x >> 4, ib = cur.eb.x >> 4;
        // the partial is stored unnormalised (sum of weight x value); the merge divides by the sum
        // of the weights
        if (r < cur.rows) {
            const size_t slot = ((size_t)ia * H + cur.h) * kSel + (cur.ea.x & 15);
            uint32_t *dst = reinterpret_cast<uint32_t *>(part_o + slot * kD) + t;
            float unused = 0.f;
#pragma unroll
            for (int n = 0; n < 16; ++n) st_u32_pol(dst + 4 * n, pack_bf16(o[n][0], o[n][1], unused), pol_part);
            if (t == 0) st_f2_pol(part_ml + slot * 2, ma, la, pol_part);
        }
        if (r + 8 < cur.rows) {
            const size_t slot = ((size_t)ib * H + cur.h) * kSel + (cur.eb.x & 15);
            uint32_t *dst = reinterpret_cast<uint32_t *>(part_o + slot * kD) + t;
            float unused = 0.f;
#pragma unroll
            for (int n = 0; n < 16; ++n) st_u32_pol(dst + 4 * n, pack_bf16(o[n][2], o[n][3], unused), pol_part);
            if (t == 0) st_f2_pol(part_ml + slot * 2, mb, lb, pol_part);
        }
        cur = nxt;
        if (cur.w >= 0) nxt = load_unit(take(), n_work, H, items, list, r);
    }
    cp_async_wait_all();
    if (blockIdx.x == 0 && threadIdx.x == 0) pdl_wait();   // the local-window kernel is complete
}

// ------------------------------------------------------------------ host side
namespace {
// Items of 16 entries: at most one partly filled item per block that was selected at all.
size_t item_bound(int n_q, int max_blocks) {
    const size_t n_entries = (size_t)n_q * kSel;
    return n_entries / kItemRows + (n_entries < (size_t)max_blocks ? n_entries : (size_t)max_blocks) + 1;
}
}  // namespace

size_t prefill_attn_workspace(int n_q, int H, int max_blocks, PrefillAttnWs *w) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    size_t off = 0;
    PrefillAttnWs l{};
    l.counts_off = off;
    off += up((size_t)max_blocks * 4);
    l.fill_off = off;
    off += up((size_t)max_blocks * 4);
    l.sched_off = off;   // the scoring GEMM's work-unit counter
    off += up(4);
    l.blk_sched_off = off;   // the block kernel's work-unit counter
    off += up(4);
    l.zero_bytes = off;
    l.n_items_off = off;
    off += up(4);
    l.items_off = off;
    off += up(item_bound(n_q, max_blocks) * sizeof(int4));
    l.list_off = off;
    off += up((size_t)n_q * kSel * sizeof(int2));
    l.sel_off = off;     // the block kernel's entries of the selection (classified)
    off += up((size_t)n_q * kSel * 4);
    l.loc_off = off;     // per query: the local blocks the tensor-core local kernel attends
    off += up((size_t)n_q * 4);
    l.tile_off = off;    // per 128-query tile: its local window {first block, blocks}
    off += up((size_t)prefill_local_tiles(n_q) * sizeof(int2));
    l.ml_off = off;
    off += up((size_t)n_q * H * kSel * 2 * 4);
    l.o_off = off;
    off += up((size_t)n_q * H * kSel * kD * 2);
    l.loc_ml_off = off;   // the local window's (m, l) per (query, head)
    off += up((size_t)n_q * H * sizeof(float2));
    l.loc_o_off = off;    // the local window's unnormalised output per (query, head), bf16
    off += up((size_t)n_q * H * kD * 2);
    if (w) *w = l;
    return off;
}

cudaError_t launch_prefill_attn(const LaunchCtx &c, const void *q, const void *k, const void *v,
                                const int32_t *bt_row, const int32_t *seq_len_ptr, const int32_t *q_pos,
                                const int32_t *sel, int n_q, int H, int max_blocks, int num_pages, float scale,
                                void *out, void *ws, int32_t *dev_err) {
    PrefillAttnWs w;
    prefill_attn_workspace(n_q, H, max_blocks, &w);
    char *base = (char *)ws;
    int32_t *counts = (int32_t *)(base + w.counts_off);
    int32_t *fill = (int32_t *)(base + w.fill_off);
    int32_t *n_items = (int32_t *)(base + w.n_items_off);
    int4 *items = (int4 *)(base + w.items_off);
    int2 *list = (int2 *)(base + w.list_off);
    int32_t *sel_ws = (int32_t *)(base + w.sel_off);
    int32_t *loc = (int32_t *)(base + w.loc_off);
    int2 *tiles = (int2 *)(base + w.tile_off);
    float *ml = (float *)(base + w.ml_off);
    __nv_bfloat16 *part_o = (__nv_bfloat16 *)(base + w.o_off);
    const int n_entries = n_q * kSel;

    // classify the selection: local-window entries to the tensor-core kernel, the rest to the
    // block kernel (after a preceding kernel of the same call, or a memset)
    cudaError_t e = launch_prefill_classify(c, sel, q_pos, seq_len_ptr, n_q, max_blocks, sel_ws, counts, loc, tiles,
                                            dev_err);
    if (e != cudaSuccess) return e;

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // every kernel here follows another kernel of the same call

    cfg.gridDim = dim3((unsigned)((n_entries + kInvThreads * kInvEntries - 1) / (kInvThreads * kInvEntries)));
    cfg.blockDim = dim3(kInvThreads);
    e = cudaLaunchKernelEx(&cfg, prefill_invert_kernel, (const int32_t *)counts, bt_row, (const int32_t *)sel_ws,
                           q_pos, n_entries, max_blocks, fill, items, n_items, list);
    if (e != cudaSuccess) return e;

    // the local windows on tcgen05, on a few SMs beside the block kernel that follows
    void *loc_o = base + w.loc_o_off;
    float2 *loc_ml = (float2 *)(base + w.loc_ml_off);
    e = launch_prefill_local(c, q, k, v, bt_row, q_pos, loc, tiles, n_q, H, num_pages, scale, loc_o, loc_ml, dev_err);
    if (e != cudaSuccess) return e;

    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_block_mma_kernel, kMmaWarps * 32, 0);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)(c.num_sms * (per_sm > 0 ? per_sm : 1)));
    cfg.blockDim = dim3(kMmaWarps * 32);
    e = cudaLaunchKernelEx(&cfg, prefill_block_mma_kernel, (const uint4 *)q, (const uint4 *)k, (const uint4 *)v,
                           (const int2 *)list, (const int4 *)items, (const int32_t *)n_items,
                           (int32_t *)(base + w.blk_sched_off), H, num_pages, scale * kLog2e, part_o, ml, dev_err);
    if (e != cudaSuccess) return e;

    return launch_prefill_merge(c, sel_ws, part_o, ml, loc_o, loc_ml, n_q, H, out);
}

}  // namespace uocr
