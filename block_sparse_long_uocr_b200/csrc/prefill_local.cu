// prefill_local.cu -- the local window of a prefill chunk on the tcgen05 tensor
// cores, and the merge of every query's partial softmax states.
//
// Unlimited-OCR-2 walk-through (news.rkmt.cn/news/25027), section 五 steps 3-4:
// every query keeps its 4 local blocks (the block holding its position and the
// 3 before it) next to its 12 remote blocks, and attends exactly over the
// selected tokens.  In a prefill chunk (release report, leheavengame.com,
// section 三: chunks of consecutive new tokens) the 128 queries of 4
// consecutive 32-token blocks share one window of 7 key blocks, so their local
// attention is a dense contraction:
//   S = Q [128 x 128] . K_win^T [128 x 224]        (tcgen05, fp32 in TMEM)
//   P = masked softmax rows of S (each row keeps its own 4 blocks, t <= p)
//   O = P [128 x 224] . V_win [224 x 128]          (tcgen05, fp32 in TMEM)
// with the causal and window mask applied while S is read back.  The remote
// blocks of the same queries are attended block by block (prefill_attn.cu).
// Each leaves one partial state per (query, slot, head) in the workspace: the
// row maximum m and weight sum l in fp32 and the unnormalised output in bf16;
// the local window's state goes to the slot of the query's first local entry.
//
// Kernels:
//   prefill_classify_kernel   one CTA per 128-query tile: validates the
//       selection (flags UOCR_DEVERR_SEL / UOCR_DEVERR_POS), decides whether
//       the tile's local windows fit one window of at most 8 blocks (always
//       for consecutive positions; otherwise the tile's local entries go to the
//       block kernel like remote ones), and splits each query's entries: the
//       first occurrence of each local block to the local kernel (a 4-bit mask
//       per query and the slot its state goes to, marked -2 in the classified
//       selection), the rest to the block kernel (block ids in the classified
//       selection, counted per block for the inversion);
//   prefill_local_kernel   persistent on a quarter of the SMs (one CTA per
//       SM), each CTA looping over an equal share of the (tile, head) units
//       while the block kernel runs on the rest, 288 threads: warp 8
//       allocates 256 TMEM columns, loads Q (two 64-dim halves, 128-byte
//       swizzle) and the window's K and V tiles (one 32-token box per block and
//       half; a page outside the pool is loaded out of bounds, i.e. as zeros,
//       and masked) with TMA, and one of its threads issues the MMAs; warps w
//       and w + 4 share TMEM lane quarter w % 4 (row = query), each taking
//       every other window block: they read S back twice (row maximum, then
//       weights), write P as bf16 into the K tile's shared memory in the
//       128-byte-swizzled K-major layout of an MMA operand, and after P V read
//       O back (64 dims each) and store it with TMA into the row's partial;
//   prefill_merge_kernel   persistent, half a warp per (query, head): every
//       valid slot's partial and the local window's state, out = sum_k
//       2^(m_k - M) acc_k / sum_k 2^(m_k - M) l_k in bf16.
// P V takes V as an MN-major operand (the V tile is token-major, dims
// contiguous), so no transpose is needed.  Weights are rounded to bf16 for the
// tensor cores and l sums the rounded weights (the output moves by at most
// ~2^-9 times the range of the values).  Every mbarrier wait is bounded in wall
// time; on a timeout the CTA flags UOCR_DEVERR_TIMEOUT, stores empty local
// states (m = -inf, which the merge skips), drains its copies and MMAs, and ends.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace uocr {

namespace {

constexpr int kTileQ = 128;                    // queries per local tile (TMEM lanes)
constexpr int kMaxWinBlocks = 8;               // key blocks of a tile's window: 7 for 4 aligned query blocks
constexpr int kMaxWinSpan = kMaxWinBlocks - 4; // largest (last - first) query block of a tile with local work
constexpr int kRowWarps = 8;                   // two per TMEM lane quarter, each with half the window's blocks
constexpr int kLocThreads = 32 * (kRowWarps + 1);   // + 1 TMA / MMA warp
constexpr int kIssueWarp = kRowWarps;
constexpr uint32_t kTmemCols = 256;            // S (up to 256 columns), then O over its first 128
constexpr int kWinBytes = kMaxWinBlocks * kBlock * 128;   // one 64-dim half of the window's K or V: 32 KiB
constexpr int kPRegionBytes = kTileQ * 128;               // 64 keys of P for 128 rows: 16 KiB
constexpr int kLocalSlotMark = -2;   // classified selection: this slot holds the local window's state
constexpr int kMergeWarps = 8;

struct __align__(1024) LocSmem {
    uint8_t q[2][kTileQ * 128];     // Q tile, two 64-dim halves, K-major SW128 (32 KiB)
    uint8_t k[2][kWinBytes];        // K of the window, two halves, K-major SW128; P over it after S
    uint8_t v[2][kWinBytes];        // V of the window, two 64-dim halves (MN-major operand), SW128
    float red_m[2][kTileQ], red_l[2][kTileQ];   // each row's maximum and weight sum over each warp half
    int red_ok[2][kTileQ];                      // each warp half's P V completed
    uint64_t bar_qk, bar_v, bar_s, bar_p, bar_o;
    uint32_t tmem_base;
    int abort_flag;
};

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle: 64 elements (128 B)
// along MN per row, rows (the K index) 128 B apart, 8-row groups 1024 B apart (SBO), the next
// 64 MN elements `mn_stride` bytes further (LBO), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t mn_stride) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)((mn_stride >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

// Shared -> global tile store (the box of `map` at (x, y, z)), tracked by this thread's bulk group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, int x, int y, int z, const void *src) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z), "r"(smem_addr(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until this thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and until they are complete (written to global memory).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Generic-proxy writes to shared memory made visible to the tensor cores (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2^x by the hardware's approximate exponential instruction (its error is far below the bf16
// rounding of the weights that follows; inputs are <= 0 here, and very negative ones give 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi, float &sum) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    sum += __low2float(v) + __high2float(v);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Drops a 128-byte line from L2 without writing it back (its contents become undefined).
__device__ __forceinline__ void l2_discard_line(const void *p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, LocSmem &s, int32_t *dev_err) {
    if (mbar_wait_timed(bar, parity, kWaitLimitNs, &s.abort_flag)) return true;
    if (atomicExch(&s.abort_flag, 1) == 0) flag_error(dev_err, UOCR_DEVERR_TIMEOUT);
    return false;
}

}  // namespace

// One CTA per tile of 128 queries; thread = query.  See the file comment.
__global__ void __launch_bounds__(kTileQ)
prefill_classify_kernel(const int32_t *__restrict__ sel, const int32_t *__restrict__ q_pos,
                        const int32_t *__restrict__ seq_len_ptr, int n_q, int max_blocks,
                        int32_t *__restrict__ sel_ws, int32_t *counts, int32_t *__restrict__ loc_info,
                        int2 *__restrict__ tile_info, int32_t *dev_err) {
    __shared__ int s_lo[kTileQ / 32], s_hi[kTileQ / 32];
    pdl_wait();
    pdl_launch_dependents();   // the inversion waits for this grid before reading its output
    const int t = blockIdx.x, r = threadIdx.x, i = t * kTileQ + r;
    const int warp = r >> 5, lane = r & 31;
    const int seq_len = min(__ldg(seq_len_ptr), max_blocks * kBlock);
    const int p = i < n_q ? __ldg(q_pos + i) : -1;
    const bool valid = i < n_q && p >= 0 && p < seq_len;
    if (i < n_q && !valid) flag_error(dev_err, UOCR_DEVERR_POS);
    const int qb = valid ? p / kBlock : 0;
    int lo = __reduce_min_sync(0xffffffffu, valid ? qb : 0x7fffffff);
    int hi = __reduce_max_sync(0xffffffffu, valid ? qb : -1);
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kTileQ / 32; ++w) {
        lo = min(lo, s_lo[w]);
        hi = max(hi, s_hi[w]);
    }
    // the tile's window: from the first local block of its lowest row to its highest row's block
    const int kb0 = hi >= 0 ? max(0, lo - (kLocal - 1)) : 0;
    const int nkb = (hi >= 0 && hi - lo <= kMaxWinSpan) ? hi - kb0 + 1 : 0;
    if (r == 0) tile_info[t] = make_int2(kb0, nkb);

    int loc = 0;
    int js[kSel];   // the caller's selection is 4-byte aligned: scalar loads
#pragma unroll
    for (int k = 0; k < kSel; ++k) js[k] = i < n_q ? __ldg(sel + (size_t)i * kSel + k) : -1;
#pragma unroll
    for (int k = 0; k < kSel; ++k) {
        int j = js[k];
        if (!valid) {
            j = -1;
        } else if (j > qb) {
            flag_error(dev_err, UOCR_DEVERR_SEL);
            j = -1;
        } else if (j < 0) {
            j = -1;
        }
        if (j >= 0 && nkb > 0 && j >= qb - (kLocal - 1)) {
            const int b = j - qb + (kLocal - 1);   // 0..3
            if (!((loc >> b) & 1)) {
                // the first occurrence goes to the local kernel; the first such slot holds its state
                if (loc == 0) loc = k << 8;
                loc |= 1 << b;
                js[k] = (loc & 0xf) == (1 << b) ? kLocalSlotMark : -1;
                continue;
            }
        }
        js[k] = j;
        if (j >= 0) atomicAdd(counts + j, 1);
    }
    if (i < n_q) {
        int4 *dst = reinterpret_cast<int4 *>(sel_ws + (size_t)i * kSel);
#pragma unroll
        for (int k = 0; k < kSel / 4; ++k) dst[k] = make_int4(js[4 * k], js[4 * k + 1], js[4 * k + 2], js[4 * k + 3]);
        loc_info[i] = loc;
    }
}

__global__ void __launch_bounds__(kLocThreads, 1)
prefill_local_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                     const int32_t *__restrict__ bt_row, const int32_t *__restrict__ q_pos,
                     const int32_t *__restrict__ loc_info, const int2 *__restrict__ tile_info, int n_units, int n_q,
                     int H, int num_pages, int q_box_rows, float scale_log2, float2 *__restrict__ loc_ml,
                     int32_t *dev_err) {
    extern __shared__ uint8_t smem_raw[];
    LocSmem &s = *reinterpret_cast<LocSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&s.bar_qk, 1);
        mbar_init(&s.bar_v, 1);
        mbar_init(&s.bar_s, 1);
        mbar_init(&s.bar_p, kRowWarps);
        mbar_init(&s.bar_o, 1);
        s.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kIssueWarp) {
        tc::tmem_alloc(&s.tmem_base, kTmemCols);
        tc::tmem_relinquish();
        if (lane == 0) {
            tc::prefetch_tensormap(&map_q);
            tc::prefetch_tensormap(&map_k);
            tc::prefetch_tensormap(&map_v);
            tc::prefetch_tensormap(&map_o);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem_base;
    // The classification (tile windows, local masks and slots) is complete once the preceding
    // kernel, the inversion, is.
    pdl_wait();
    // The block kernel that follows may start now (it reads only the inversion, complete at this
    // point) and runs beside this grid; it waits for this grid at its end, so the merge after it
    // starts once both are done.
    pdl_launch_dependents();

    int it = 0;   // units done by this CTA: each unit completes every barrier once (parity it & 1)
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int t = u / H, h = u % H;
        const int2 ti = tile_info[t];
        const int kb0 = ti.x, nkb = ti.y;
        if (nkb == 0) continue;   // uniform over the CTA
        const uint32_t ph = (uint32_t)(it & 1);
        ++it;
        if (warp == kIssueWarp) {
            // -------------------------------------------------------- TMA loads and MMAs
            if (lane == 0) {
                bulk_wait_read();   // the previous unit's O stores have read the Q tile's shared memory
                const uint32_t q_bytes = 2u * (uint32_t)q_box_rows * 128u;
                const uint32_t kv_bytes = (uint32_t)nkb * 2u * kBlock * 128u;
                mbar_arrive_expect_tx(&s.bar_qk, q_bytes + kv_bytes);
                tma_load_3d(s.q[0], &map_q, 0, h, t * kTileQ, &s.bar_qk);
                tma_load_3d(s.q[1], &map_q, 64, h, t * kTileQ, &s.bar_qk);
                // a page outside the pool is read out of bounds (zeros) and masked by the row warps
                auto tile_z = [&](int b) {
                    const int page = __ldg(bt_row + kb0 + b);
                    return (unsigned)page < (unsigned)num_pages ? page * H + h : num_pages * H;
                };
                for (int b = 0; b < nkb; ++b) {
                    const int z = tile_z(b);
                    tma_load_3d(s.k[0] + b * (kBlock * 128), &map_k, 0, 0, z, &s.bar_qk);
                    tma_load_3d(s.k[1] + b * (kBlock * 128), &map_k, 64, 0, z, &s.bar_qk);
                }
                mbar_arrive_expect_tx(&s.bar_v, kv_bytes);
                for (int b = 0; b < nkb; ++b) {
                    const int z = tile_z(b);
                    tma_load_3d(s.v[0] + b * (kBlock * 128), &map_v, 0, 0, z, &s.bar_v);
                    tma_load_3d(s.v[1] + b * (kBlock * 128), &map_v, 64, 0, z, &s.bar_v);
                }
                bool issued_s = false, issued_o = false, ok = false;
                if (wait_or_abort(&s.bar_qk, ph, s, dev_err)) {
                    tc::fence_after_sync();
                    // S = Q K^T: M = 128 rows, N = 32 nkb keys, 8 k-steps of 16 dims (32 bytes into a
                    // 128-byte swizzle row: 2 in the descriptor's 16-byte address field)
                    const uint32_t idesc_s = tc::idesc_bf16_f32(kTileQ, nkb * kBlock);
                    const uint64_t qd0 = tc::smem_desc_k_sw128(smem_addr(s.q[0]));
                    const uint64_t qd1 = tc::smem_desc_k_sw128(smem_addr(s.q[1]));
                    const uint64_t kd0 = tc::smem_desc_k_sw128(smem_addr(s.k[0]));
                    const uint64_t kd1 = tc::smem_desc_k_sw128(smem_addr(s.k[1]));
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint64_t koff = (uint64_t)((k & 3) * 2);
                        tc::mma_bf16(tmem, (k < 4 ? qd0 : qd1) + koff, (k < 4 ? kd0 : kd1) + koff, idesc_s,
                                     k > 0 ? 1u : 0u);
                    }
                    tc::commit(&s.bar_s);
                    issued_s = true;
                    // O = P V: P [128 x 32 nkb] K-major in 64-key regions of 16 KiB over the K tile; V
                    // the MN-major operand (dims contiguous), 16 keys = two 8-row groups = 2 KiB per
                    // k-step, its two 64-dim halves kWinBytes apart
                    if (wait_or_abort(&s.bar_p, ph, s, dev_err) && wait_or_abort(&s.bar_v, ph, s, dev_err)) {
                        tc::fence_after_sync();
                        const uint32_t idesc_o = tc::idesc_bf16_f32(kTileQ, kD) | (1u << 16);   // B MN-major
                        const uint32_t p0 = smem_addr(s.k[0]), v0 = smem_addr(s.v[0]);
                        for (int st = 0; st < 2 * nkb; ++st) {
                            const uint64_t ad = tc::smem_desc_k_sw128(p0 + (uint32_t)(st >> 2) * kPRegionBytes) +
                                                (uint64_t)((st & 3) * 2);
                            const uint64_t bd = smem_desc_mn_sw128(v0 + (uint32_t)st * 2048u, (uint32_t)kWinBytes);
                            tc::mma_bf16(tmem, ad, bd, idesc_o, st > 0 ? 1u : 0u);
                        }
                        tc::commit(&s.bar_o);
                        issued_o = true;
                        ok = true;
                    }
                }
                if (!ok) {
                    // drain: the unit's copies have landed and its MMAs completed before the CTA ends
                    mbar_drain(&s.bar_qk, ph, dev_err);
                    mbar_drain(&s.bar_v, ph, dev_err);
                    if (issued_s) mbar_drain(&s.bar_s, ph, dev_err);
                    if (issued_o) mbar_drain(&s.bar_o, ph, dev_err);
                }
            }
            __syncwarp();
        } else {
            // -------------------------------------------------------- row warps: softmax, partial
            // Warps w and w + 4 share TMEM lane quarter w % 4 (rows r = 32 (w % 4) + lane); warp half
            // hh = w / 4 takes the window blocks b with b % 2 == hh and the output dims 64 hh .. + 63.
            const int quarter = warp & 3, hh = warp >> 2;
            const int r = quarter * 32 + lane;
            const int i = t * kTileQ + r;
            const bool row_ok = i < n_q;
            // the row's position and local mask and the window's pages, loaded while the unit's
            // tiles and S are on their way (pinned: not sunk past the wait below)
            const int p = row_ok ? ld_pinned(q_pos + i) : -1;
            const int li = row_ok ? ld_pinned(loc_info + i) : 0;
            int pages[kMaxWinBlocks];
#pragma unroll
            for (int b = 0; b < kMaxWinBlocks; ++b) pages[b] = b < nkb ? ld_pinned(bt_row + kb0 + b) : 0;
            const int loc = li & 0xf;
            const int qb = p >= 0 ? p / kBlock : 0;
            const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
            // pages of the window inside the pool (the same test as the loads)
            unsigned pmask = 0;
#pragma unroll
            for (int b = 0; b < kMaxWinBlocks; ++b) {
                if (b >= nkb) continue;
                if ((unsigned)pages[b] < (unsigned)num_pages)
                    pmask |= 1u << b;
                else if (threadIdx.x == 0 && h == 0)
                    flag_error(dev_err, UOCR_DEVERR_PAGE);
            }
            // window block b is one of this row's local blocks (bit d = kb0 + b - (qb - 3) of loc)
            auto in_row = [&](int b) {
                const int d = kb0 + b - qb + (kLocal - 1);
                return b < nkb && d >= 0 && d < kLocal && ((loc >> d) & 1) && ((pmask >> b) & 1);
            };
            // a warp-uniform verdict on a wait (tcgen05.ld is warp-collective)
            auto warp_wait = [&](uint64_t *bar) {
                return __all_sync(0xffffffffu, wait_or_abort(bar, ph, s, dev_err));
            };
            // the pair's named barrier (ids 1..4; 0 is __syncthreads)
            auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory"); };
            // Both warps of a pair pass both pair barriers whatever their waits return, so that a
            // timeout in one cannot leave the other at a barrier.
            float m = -INFINITY, l = 0.f, mh = -INFINITY, lh = 0.f;
            bool have_o = false;
            const bool ok_s = warp_wait(&s.bar_s);
            unsigned need = 0;   // this warp's blocks that some row of the quarter keeps (warp-uniform)
            if (ok_s) {
                tc::fence_after_sync();
#pragma unroll
                for (int b2 = 0; b2 < kMaxWinBlocks / 2; ++b2)
                    if (__any_sync(0xffffffffu, in_row(2 * b2 + hh))) need |= 1u << b2;
                // pass 1: the maximum of z = scale * log2(e) * s over the row's visible tokens (the
                // causal test only on the block that holds the row's position)
#pragma unroll
                for (int b2 = 0; b2 < kMaxWinBlocks / 2; ++b2) {
                    if (!((need >> b2) & 1)) continue;
                    const int b = 2 * b2 + hh;
                    float v[32];
                    tc::tmem_ld_32x32b_x32(trow + (uint32_t)(b * kBlock), v);
                    tc::tmem_ld_wait();
                    if (in_row(b)) {
                        const int t0 = (kb0 + b) * kBlock;
                        float bm = -INFINITY;
                        if (t0 + kBlock - 1 <= p) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) bm = fmaxf(bm, v[c]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (t0 + c <= p) bm = fmaxf(bm, v[c]);
                        }
                        // scale * log2(e) may be negative (a caller's scale): the extreme of s that
                        // maximises z
                        if (scale_log2 < 0.f) {
                            bm = INFINITY;
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (t0 + c <= p) bm = fminf(bm, v[c]);
                        }
                        mh = fmaxf(mh, bm * scale_log2);
                    }
                }
            }
            s.red_m[hh][r] = mh;
            pair_sync();
            m = fmaxf(mh, s.red_m[hh ^ 1][r]);
            if (ok_s) {
                // pass 2: weights 2^(z - m), rounded to bf16, into P (zeros outside the row's blocks)
#pragma unroll
                for (int b2 = 0; b2 < kMaxWinBlocks / 2; ++b2) {
                    const int b = 2 * b2 + hh;
                    if (b >= nkb) continue;
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) pk[c] = 0u;
                    if ((need >> b2) & 1) {
                        float v[32];
                        tc::tmem_ld_32x32b_x32(trow + (uint32_t)(b * kBlock), v);
                        tc::tmem_ld_wait();
                        if (in_row(b)) {
                            const int t0 = (kb0 + b) * kBlock;
                            const float nm = -m;
                            if (t0 + kBlock - 1 <= p) {
#pragma unroll
                                for (int c = 0; c < 16; ++c)
                                    pk[c] = pack2_bf16(ex2_approx(fmaf(v[2 * c], scale_log2, nm)),
                                                       ex2_approx(fmaf(v[2 * c + 1], scale_log2, nm)), lh);
                            } else {
#pragma unroll
                                for (int c = 0; c < 16; ++c) {
                                    const float e0 = t0 + 2 * c <= p ? ex2_approx(fmaf(v[2 * c], scale_log2, nm)) : 0.f;
                                    const float e1 =
                                        t0 + 2 * c + 1 <= p ? ex2_approx(fmaf(v[2 * c + 1], scale_log2, nm)) : 0.f;
                                    pk[c] = pack2_bf16(e0, e1, lh);
                                }
                            }
                        }
                    }
                    // keys 32 b .. 32 b + 31 of row r: region (32 b) / 64, 16-byte chunks (32 b % 64) / 8 + u,
                    // stored at chunk ^ (r % 8) of the row's 128 bytes
                    uint8_t *row_base = s.k[0] + (size_t)((b * kBlock) >> 6) * kPRegionBytes + (size_t)r * 128;
                    const int c0 = ((b * kBlock) & 63) >> 3;
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4)
                        *reinterpret_cast<uint4 *>(row_base + (((c0 + u4) ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * u4], pk[4 * u4 + 1], pk[4 * u4 + 2], pk[4 * u4 + 3]);
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.bar_p);
                if (warp_wait(&s.bar_o)) {
                    tc::fence_after_sync();
                    have_o = true;
                }
            }
            s.red_l[hh][r] = lh;
            s.red_ok[hh][r] = have_o ? 1 : 0;
            pair_sync();
            l = lh + s.red_l[hh ^ 1][r];
            const bool pair_ok = have_o && s.red_ok[hh ^ 1][r] != 0;
            // the row's local state: unnormalised O in bf16 (this warp's 64 dims) into the Q tile's
            // half hh (the box layout of the local-partial map: row r at 128 r, chunk c at c ^ (r % 8)),
            // stored below by TMA; (m, l) in fp32; an empty state (m = -inf) after a timeout
            if (pair_ok) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float o[32];
                    tc::tmem_ld_32x32b_x32(trow + (uint32_t)(hh * 64 + c * 32), o);
                    tc::tmem_ld_wait();
                    float unused = 0.f;
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        *reinterpret_cast<uint4 *>(s.q[hh] + r * 128 + (((c * 4 + x) ^ (r & 7)) << 4)) =
                            make_uint4(pack2_bf16(o[8 * x], o[8 * x + 1], unused),
                                       pack2_bf16(o[8 * x + 2], o[8 * x + 3], unused),
                                       pack2_bf16(o[8 * x + 4], o[8 * x + 5], unused),
                                       pack2_bf16(o[8 * x + 6], o[8 * x + 7], unused));
                }
                fence_proxy_async_smem();   // visible to the TMA store
            } else {
                m = -INFINITY;
                l = 0.f;
            }
            if (row_ok && loc != 0 && hh == 0) loc_ml[(size_t)i * H + h] = make_float2(m, l);
        }
        // the unit's TMEM reads and MMAs are complete before the next unit's overwrite them
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (warp == kIssueWarp && lane == 0) {
            // the tile's O rows of head h (rows past n_q are clipped by the store; a row whose state
            // is empty or that has no local entries is stored too and never read)
            tma_store_3d(&map_o, 0, h, t * kTileQ, s.q[0]);
            tma_store_3d(&map_o, 64, h, t * kTileQ, s.q[1]);
            bulk_commit();
        }
        if (*(volatile int *)&s.abort_flag) break;
    }
    if (warp == kIssueWarp && lane == 0) bulk_wait_all();   // the last stores are complete

    tc::fence_before_sync();
    __syncthreads();
    if (warp == kIssueWarp) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// Half a warp per (query, head): lane k of the half holds slot k's (m, l) and output dims 8 k ..
// 8 k + 7 of every partial.  A slot holds a block partial when the classified selection names a
// block there; the local window's state, when the query has one, is a seventeenth partial.  Empty
// states (m = -inf, after a timeout) are skipped.  Persistent: warp w of the grid takes the pairs
// of (query, head)s 2 w, 2 w + 1, then 2 (w + warps), ..., and loads the next pair's entries and
// (m, l) while the current pair's partials are on their way.  n_q * H < 2^31 (checked by the
// launcher).
__global__ void __launch_bounds__(kMergeWarps * 32)
prefill_merge_kernel(const int32_t *__restrict__ sel_ws, const __nv_bfloat16 *__restrict__ part_o,
                     const float *__restrict__ part_ml, const __nv_bfloat16 *__restrict__ loc_o,
                     const float2 *__restrict__ loc_ml, int n_q, int H, __nv_bfloat16 *__restrict__ out) {
    const int k = threadIdx.x & 15;
    const unsigned half = 0xffffu << (threadIdx.x & 16);   // this half-warp's lanes
    const int n = n_q * H;
    const int stride = 2 * gridDim.x * kMergeWarps;
    // A half past the end repeats the last (query, head) and stores nothing, so that every lane
    // takes part in the warp's shuffles and both halves run the same iterations.
    auto clamp = [&](int ih) { return ih < n ? ih : n - 1; };
    // the first round of a (query, head)'s loads: the slot's entry, its (m, l) and the local
    // state's (m, l) (the (m, l) line of a (query, head) is read whole either way; an unnamed
    // slot's value is not used)
    struct First {
        int js;
        float2 ml, mll;
    };
    auto first = [&](int ih) {
        First f;
        f.js = __ldg(sel_ws + (size_t)(ih / H) * kSel + k);
        f.ml = __ldcs(reinterpret_cast<const float2 *>(part_ml) + (size_t)ih * kSel + k);
        f.mll = __ldcs(loc_ml + ih);
        return f;
    };
    int pair = blockIdx.x * (2 * kMergeWarps) + (threadIdx.x >> 5) * 2;   // even (query, head) of the warp
    pdl_wait();
    if (pair >= n) return;   // uniform over the warp
    int ih = clamp(pair + ((threadIdx.x >> 4) & 1));
    First cur = first(ih);
    for (; pair < n; pair += stride) {
        const bool live = pair + ((threadIdx.x >> 4) & 1) < n;
        const size_t base = (size_t)ih * kSel;
        const bool has_loc = (__ballot_sync(0xffffffffu, cur.js == kLocalSlotMark) & half) != 0u;
        const unsigned named = (__ballot_sync(0xffffffffu, cur.js >= 0) & half) >> (threadIdx.x & 16);
        const uint4 *src = reinterpret_cast<const uint4 *>(part_o + base * kD) + k;
        uint4 v[kSel];
#pragma unroll
        for (int s = 0; s < kSel; ++s)
            v[s] = (named >> s & 1u) ? __ldcs(src + s * (kD / 8)) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 vl = has_loc ? __ldcs(reinterpret_cast<const uint4 *>(loc_o + (size_t)ih * kD) + k)
                                 : make_uint4(0u, 0u, 0u, 0u);
        // the next pair's first round, in flight beside this pair's partials
        const int ih_next = clamp(pair + stride + ((threadIdx.x >> 4) & 1));
        const First nxt = pair + stride < n ? first(ih_next) : cur;
        // a named slot with m = -inf (an empty state) and a missing local state are skipped
        const float2 mlv = cur.js >= 0 ? cur.ml : make_float2(-INFINITY, 0.f);
        const float2 mll = has_loc ? cur.mll : make_float2(-INFINITY, 0.f);
        const unsigned vmask = (__ballot_sync(0xffffffffu, mlv.x != -INFINITY) & half) >> (threadIdx.x & 16);
        const bool loc_ok = mll.x != -INFINITY;
        float M = fmaxf(mlv.x, mll.x);
#pragma unroll
        for (int x = 8; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x, 16));
        // partial s holds sum_t 2^(z_t - m_s) v_t and l_s = sum_t 2^(z_t - m_s): rescale both to M
        const float w = mlv.x != -INFINITY ? exp2f(mlv.x - M) : 0.f;
        const float wl = loc_ok ? exp2f(mll.x - M) : 0.f;
        float W = mlv.y * w;
#pragma unroll
        for (int x = 8; x > 0; x >>= 1) W += __shfl_xor_sync(0xffffffffu, W, x, 16);
        W += mll.y * wl;
        float A[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        auto acc = [&](float ws, const uint4 &u) {
            A[0] = fmaf(ws, __uint_as_float(u.x << 16), A[0]);
            A[1] = fmaf(ws, __uint_as_float(u.x & 0xffff0000u), A[1]);
            A[2] = fmaf(ws, __uint_as_float(u.y << 16), A[2]);
            A[3] = fmaf(ws, __uint_as_float(u.y & 0xffff0000u), A[3]);
            A[4] = fmaf(ws, __uint_as_float(u.z << 16), A[4]);
            A[5] = fmaf(ws, __uint_as_float(u.z & 0xffff0000u), A[5]);
            A[6] = fmaf(ws, __uint_as_float(u.w << 16), A[6]);
            A[7] = fmaf(ws, __uint_as_float(u.w & 0xffff0000u), A[7]);
        };
        if (loc_ok) acc(wl, vl);   // (an empty local state's output is not read: it may be anything)
#pragma unroll
        for (int s = 0; s < kSel; ++s) {
            const float ws = __shfl_sync(0xffffffffu, w, s, 16);
            if (vmask >> s & 1u) acc(ws, v[s]);
        }
        // Every lane of the warp has used its loads' values: drop this (query, head)'s partial
        // lines from L2 (its 16 x 256 bytes of outputs are 32 lines, two per lane; its 16 (m, l)
        // pairs one line; its local output two), so that they are never written back.  The
        // workspace is 256-byte aligned, so the lines belong to this (query, head) alone; a slot
        // not written in this call holds nothing that is needed.
        __syncwarp();
        if (live) {
            const char *po = reinterpret_cast<const char *>(part_o + base * kD);
            l2_discard_line(po + 256 * k);
            l2_discard_line(po + 256 * k + 128);
            if (k == 0) l2_discard_line(part_ml + base * 2);
            if (has_loc && k < 2)
                l2_discard_line(reinterpret_cast<const char *>(loc_o + (size_t)ih * kD) + 128 * k);
            const float inv = W > 0.f ? 1.f / W : 0.f;
            float unused = 0.f;
            uint4 pk;
            pk.x = pack2_bf16(A[0] * inv, A[1] * inv, unused);
            pk.y = pack2_bf16(A[2] * inv, A[3] * inv, unused);
            pk.z = pack2_bf16(A[4] * inv, A[5] * inv, unused);
            pk.w = pack2_bf16(A[6] * inv, A[7] * inv, unused);
            reinterpret_cast<uint4 *>(out + (size_t)ih * kD)[k] = pk;
        }
        ih = ih_next;
        cur = nxt;
    }
}

// ---------------------------------------------------------------- host side
size_t prefill_local_smem() { return sizeof(LocSmem) + 1024; }

int prefill_local_tiles(int n_q) { return (n_q + kTileQ - 1) / kTileQ; }

cudaError_t launch_prefill_classify(const LaunchCtx &c, const int32_t *sel, const int32_t *q_pos,
                                    const int32_t *seq_len_ptr, int n_q, int max_blocks, int32_t *sel_ws,
                                    int32_t *counts, int32_t *loc_info, int2 *tile_info, int32_t *dev_err) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)prefill_local_tiles(n_q));
    cfg.blockDim = dim3(kTileQ);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, prefill_classify_kernel, sel, q_pos, seq_len_ptr, n_q, max_blocks, sel_ws, counts,
                              loc_info, tile_info, dev_err);
}

bool prefill_kv_tensor_map(CUtensorMap *map, const void *cache, int num_pages, int H) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)kBlock, (cuuint64_t)num_pages * H};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kBlock * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kBlock, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(cache), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_prefill_local(const LaunchCtx &c, const void *q, const void *k, const void *v,
                                 const int32_t *bt_row, const int32_t *q_pos, const int32_t *loc_info,
                                 const int2 *tile_info, int n_q, int H, int num_pages, float scale, void *loc_o,
                                 float2 *loc_ml, int32_t *dev_err) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorInvalidValue;
    const int q_box_rows = n_q < kTileQ ? n_q : kTileQ;
    CUtensorMap map_q, map_k, map_v, map_o;
    // q [n_q][H][128] and the local partials [n_q][H][128]: dims (dim, head, query), one head's rows
    // of a tile per box
    for (int which = 0; which < 2; ++which) {
        const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)n_q};
        const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
        const cuuint32_t box[3] = {64, 1, (cuuint32_t)q_box_rows};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (enc(which ? &map_o : &map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, which ? loc_o : const_cast<void *>(q),
                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (!prefill_kv_tensor_map(&map_k, k, num_pages, H) || !prefill_kv_tensor_map(&map_v, v, num_pages, H))
        return cudaErrorInvalidValue;
    const long long units = (long long)prefill_local_tiles(n_q) * H;
    if (units > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const size_t smem = prefill_local_smem();
    cudaError_t e = cudaFuncSetAttribute(prefill_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    // A quarter of the SMs (one CTA each: the kernel holds most of an SM's shared memory), each
    // taking the same number of units; the block kernel launched after this one fills the rest.
    const long long share = c.num_sms / 4 > 0 ? c.num_sms / 4 : 1;
    const long long per_cta = (units + share - 1) / share;
    const long long ctas = per_cta > 0 ? (units + per_cta - 1) / per_cta : 0;
    cfg.gridDim = dim3((unsigned)(ctas > 0 ? ctas : 1));
    cfg.blockDim = dim3(kLocThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // always after the classification of the same call
    return cudaLaunchKernelEx(&cfg, prefill_local_kernel, map_q, map_k, map_v, map_o, bt_row, q_pos, loc_info,
                              tile_info, (int)units, n_q, H, num_pages, q_box_rows, scale * kLog2e, loc_ml, dev_err);
}

cudaError_t launch_prefill_merge(const LaunchCtx &c, const int32_t *sel_ws, const void *part_o, const float *part_ml,
                                 const void *loc_o, const float2 *loc_ml, int n_q, int H, void *out) {
    if ((long long)n_q * H > 0x7fffffffLL / 2) return cudaErrorInvalidConfiguration;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_merge_kernel, kMergeWarps * 32, 0);
    if (e != cudaSuccess) return e;
    // persistent: as many CTAs as fit at once, fewer when there are fewer pairs
    const long long need = ((long long)n_q * H + 2 * kMergeWarps - 1) / (2 * kMergeWarps);
    const long long fit = (long long)c.num_sms * (per_sm > 0 ? per_sm : 1);
    const long long merge_ctas = need < fit ? need : fit;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)merge_ctas);
    cfg.blockDim = dim3(kMergeWarps * 32);
    cfg.stream = c.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // always after the block kernel of the same call
    return cudaLaunchKernelEx(&cfg, prefill_merge_kernel, sel_ws, (const __nv_bfloat16 *)part_o, part_ml,
                              (const __nv_bfloat16 *)loc_o, loc_ml, n_q, H, (__nv_bfloat16 *)out);
}

}  // namespace uocr
