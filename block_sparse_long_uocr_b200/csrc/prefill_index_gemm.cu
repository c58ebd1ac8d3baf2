// prefill_index_gemm.cu -- chunked-prefill block scoring on the tcgen05 tensor cores.
//
// Unlimited-OCR-2 release report (leheavengame.com, "百度OCR-2开源", section 三): a
// prefill chunk of `tokens` queries builds a [tokens, context/32] block-score
// tensor.  With many queries per sequence the indexer scan becomes a dense
// contraction, S = Qi [n_q x 128] . Ki^T [128 x tokens], followed by the block
// maximum of the walk-through (news.rkmt.cn/news/25027, section 五 step 2):
//   scores[i][j] = max_{t in block j, t <= p_i} S[i][t].
//
// Kernel (persistent, one CTA per SM, 384 threads, warp-specialised).  A CTA
// tile is two 128-query subtiles that share every key tile they load, which
// halves the key traffic from L2 per FLOP against one subtile per CTA:
//   warp 8  TMA producer of queries: per work unit the two 128-query A subtiles
//           (two 64-dim halves each, 128-byte swizzle) into a 2-deep ring;
//   warp 10 TMA producer of keys: per 128-token N tile the 4 pages' indexer
//           keys (8 boxes of 32 tokens x 64 dims, gathered through the block
//           table) into a 3-stage ring.  The two producers run ahead of the MMAs
//           independently, each as far as its ring allows;
//   warps 9, 11  MMA issuers, one per subtile: warp 9 allocates 512 TMEM columns
//           (two buffers x two subtiles of 128 x 128 fp32); each issues 8
//           tcgen05.mma (M=128, N=128, K=16) per tile into its subtile's
//           accumulator, so that one thread's barrier waits and commits overlap
//           the other's MMAs and the tensor pipe does not drain between tiles;
//   warps 0-7 epilogue: tcgen05.ld of the accumulators (warp w owns rows
//           32(w%4) .. +31 = its TMEM lane quarter, of subtile w/4, and the
//           tile's 4 blocks), max over each 32-column block (the causal mask only
//           on blocks that reach past the row's position), fp32 scores to global
//           memory, four at a time.
// Work unit = (256-query tile, chunk of 4 N tiles); units whose tokens all lie
// past the tile's last query are skipped.  The query producer picks the CTA's
// units (from a per-launch queue when one is given, else round-robin) and
// publishes each with its A stage -- shape, page ids -- for every other role.  Every mbarrier wait is bounded in
// wall time: on timeout the CTA reports UOCR_DEVERR_TIMEOUT, every role stops
// issuing, waits (bounded) for what it issued, and the TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace uocr {

namespace {

constexpr int kBM = 128;                  // queries per subtile (TMEM lanes)
constexpr int kMT = 2;                    // subtiles per CTA tile (they share each key tile)
constexpr int kBN = 128;                  // tokens per N tile (4 pages)
constexpr int kPagesPerTile = kBN / kBlock;
constexpr int kTilesPerUnit = 4;
constexpr int kStagesB = 3;
constexpr int kStagesA = 2;
constexpr int kHalfBytesA = kBM * 128;    // one 64-dim half of an A subtile: 16 KiB
constexpr int kHalfBytesB = kBN * 128;    // one 64-dim half of a B tile: 16 KiB
constexpr int kBoxBytesB = kBlock * 128;  // one page x 64 dims: 4 KiB
constexpr int kEpiWarps = 8;             // one warp per (TMEM lane quarter, subtile)
constexpr int kProducerWarp = 8;          // query (A) tiles
constexpr int kMmaWarp = 9;               // MMA issuer of subtile 0; allocates the TMEM
constexpr int kProducerBWarp = 10;        // key (B) tiles
constexpr int kMmaWarp1 = 11;             // MMA issuer of subtile 1
constexpr int kThreads = 384;

struct __align__(1024) Smem {
    uint8_t a[kStagesA][kMT][2][kHalfBytesA];   // 128 KiB
    uint8_t b[kStagesB][2][kHalfBytesB];        // 96 KiB
    uint64_t a_full[kStagesA], a_empty[kStagesA];
    uint64_t b_full[kStagesB], b_empty[kStagesB];
    uint64_t acc_full[2][kMT], acc_empty[2][kMT];   // per accumulator buffer and subtile
    uint64_t mma_done[kMT];
    // The work unit of each A stage, written by the query producer before it arrives on desc_full
    // and read by every other role (0 tiles: no more units); the stage is rewritten only after the
    // two MMA issuers, the key producer and the 8 epilogue warps have released it (a_empty).
    uint64_t desc_full[kStagesA];
    int unit_u[kStagesA], unit_tiles[kStagesA], unit_nsub[kStagesA];
    int unit_pages[kStagesA][kTilesPerUnit * kPagesPerTile];   // -1: not loaded (outside the pool or
                                                               // past the unit's causal range)
    uint32_t tmem_base;
    int abort_flag;
};

struct UnitInfo {
    int m0;       // first query of the tile
    int nsub;     // subtiles holding queries (1 or 2)
    int t0;       // first N tile
    int ntiles;   // tiles to compute (0: skip)
    int nb_max;   // causal blocks of the tile's last valid query
};

// Same answer in every role: the unit's tile range, from the queries' positions.  Split in
// two so that a role issues the next unit's position loads (pos_prefetch: predicated loads into
// registers, nothing consumes them yet) before working on the current unit, and reduces them
// (unit_info) when it gets there: no role waits on L2 at a unit boundary.
// (ld_pinned, common.cuh: the prefetches stay where they are issued, so the memory latency is not
// put back on the unit boundary.)

struct PosPrefetch {
    int raw[kBM * kMT / 32];   // position of row m0 + 32k + lane, -1 past the queries
};
__device__ __forceinline__ PosPrefetch pos_prefetch(int u, int n_units, int n_chunks, const int32_t *q_pos,
                                                    int n_q, int lane) {
    PosPrefetch f;
    const int m0 = (u / n_chunks) * (kBM * kMT);
#pragma unroll
    for (int k = 0; k < kBM * kMT / 32; ++k) {
        const int row = m0 + k * 32 + lane;
        f.raw[k] = (u < n_units && row < n_q) ? ld_pinned(q_pos + row) : -1;
    }
    return f;
}
__device__ __forceinline__ UnitInfo unit_info(int u, int n_chunks, int n_q, int seq_len, const PosPrefetch &f) {
    UnitInfo w;
    w.m0 = (u / n_chunks) * (kBM * kMT);
    w.nsub = min(kMT, (n_q - w.m0 + kBM - 1) / kBM);
    w.t0 = (u % n_chunks) * kTilesPerUnit;
    int pmax_lane = -1;
#pragma unroll
    for (int k = 0; k < kBM * kMT / 32; ++k) pmax_lane = max(pmax_lane, f.raw[k] < seq_len ? f.raw[k] : -1);
    const int pmax = __reduce_max_sync(0xffffffffu, pmax_lane);
    w.nb_max = pmax < 0 ? 0 : pmax / kBlock + 1;
    const int tiles_needed = (w.nb_max + kPagesPerTile - 1) / kPagesPerTile;
    w.ntiles = max(0, min(kTilesPerUnit, tiles_needed - w.t0));
    return w;
}

// Lane 0 waits; the verdict is broadcast so the whole warp leaves its loops together.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, Smem &s, int32_t *dev_err, int lane,
                                          uint64_t limit_ns = kWaitLimitNs) {
    int ok = 1;
    if (lane == 0) {
        ok = mbar_wait_timed(bar, parity, limit_ns, &s.abort_flag);
        if (!ok) {
            if (!*(volatile int *)&s.abort_flag) flag_error(dev_err, UOCR_DEVERR_TIMEOUT);
            atomicExch(&s.abort_flag, 1);
        }
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Two barriers at once: both probes are issued before either result is used, so their latencies
// overlap; only a phase that is not complete yet is waited for.
__device__ __forceinline__ bool warp_wait2(uint64_t *bar0, uint32_t parity0, uint64_t *bar1, uint32_t parity1, Smem &s,
                                           int32_t *dev_err, int lane) {
    int ok = 1;
    if (lane == 0) {
        const bool r0 = mbar_try_wait(bar0, parity0);
        const bool r1 = mbar_try_wait(bar1, parity1);
        ok = (r0 || mbar_wait_timed(bar0, parity0, kWaitLimitNs, &s.abort_flag)) &&
             (r1 || mbar_wait_timed(bar1, parity1, kWaitLimitNs, &s.abort_flag));
        if (!ok) {
            if (!*(volatile int *)&s.abort_flag) flag_error(dev_err, UOCR_DEVERR_TIMEOUT);
            atomicExch(&s.abort_flag, 1);
        }
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ bool aborted(Smem &s) { return *(volatile int *)&s.abort_flag != 0; }

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
prefill_index_gemm_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                          const int32_t *__restrict__ bt_row, const int32_t *__restrict__ seq_len_ptr,
                          const int32_t *__restrict__ q_pos, int n_q, int a_box_rows, int num_pages,
                          int max_blocks, int n_chunks, int n_units, float *__restrict__ scores,
                          int32_t *sched, int32_t *dev_err, uint64_t first_wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int k = 0; k < kStagesA; ++k) {
            mbar_init(&s.a_full[k], 1);
            mbar_init(&s.a_empty[k], kMT + 1 + kEpiWarps);
            mbar_init(&s.desc_full[k], 1);
        }
        for (int k = 0; k < kStagesB; ++k) {
            mbar_init(&s.b_full[k], 1);
            mbar_init(&s.b_empty[k], kMT);
        }
        for (int k = 0; k < 2; ++k)
            for (int m = 0; m < kMT; ++m) {
                mbar_init(&s.acc_full[k][m], 1);
                mbar_init(&s.acc_empty[k][m], kEpiWarps / kMT);
            }
        for (int m = 0; m < kMT; ++m) mbar_init(&s.mma_done[m], 1);
        s.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(&s.tmem_base, 512);
        tc::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        tc::prefetch_tensormap(&map_q);
        tc::prefetch_tensormap(&map_k);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem_base;

    pdl_wait();   // inputs may come from the preceding kernel in the stream
    const int seq_len = __ldg(seq_len_ptr);
    if (threadIdx.x == 0 && seq_len > max_blocks * kBlock) flag_error(dev_err, UOCR_DEVERR_POS);
    const int seq_len_ok = min(seq_len, max_blocks * kBlock);

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer: query tiles
        // It picks the CTA's work units -- from the launch's queue when `sched` is given (a CTA that
        // runs faster takes more units), else round-robin -- one unit ahead, so that the next
        // unit's positions and page ids are in flight while the current one is published.
        int uc = 0;
        int a_fills[kStagesA] = {};
        auto pick = [&](int prev) {
            if (!sched) return prev < 0 ? (int)blockIdx.x : prev + (int)gridDim.x;
            int v = 0;
            if (lane == 0) v = atomicAdd(sched, 1);
            return __shfl_sync(0xffffffffu, v, 0);
        };
        // a unit's page ids (the block table row is read in bounds before the unit's causal range
        // is known): lane l < 4 * kTilesPerUnit holds block t0 * 4 + l
        auto unit_pages = [&](int u) {
            int pg = -1;
            if (u < n_units && lane < kTilesPerUnit * kPagesPerTile) {
                const int j = (u % n_chunks) * kTilesPerUnit * kPagesPerTile + lane;
                if (j < max_blocks) pg = ld_pinned(bt_row + j);
            }
            return pg;
        };
        int u = pick(-1);
        PosPrefetch pf = pos_prefetch(u, n_units, n_chunks, q_pos, n_q, lane);
        int pages_pf = unit_pages(u);
        int u_next = u < n_units ? pick(u) : n_units;
        while (u < n_units) {
            const UnitInfo w = unit_info(u, n_chunks, n_q, seq_len_ok, pf);
            int upage = pages_pf;
            const int u_cur = u;
            pf = pos_prefetch(u_next, n_units, n_chunks, q_pos, n_q, lane);
            pages_pf = unit_pages(u_next);
            u = u_next;
            u_next = u < n_units ? pick(u) : n_units;
            if (w.ntiles == 0) continue;
            // keep the blocks of the unit's tiles inside the causal range; flag pages outside the pool
            if (lane < w.ntiles * kPagesPerTile && w.t0 * kPagesPerTile + lane < w.nb_max) {
                if ((unsigned)upage >= (unsigned)num_pages) {
                    flag_error(dev_err, UOCR_DEVERR_PAGE);
                    upage = -1;
                }
            } else {
                upage = -1;
            }
            const int sa = uc % kStagesA;
            if (!warp_wait(&s.a_empty[sa], ((uc / kStagesA) & 1) ^ 1, s, dev_err, lane)) break;
            if (lane < kTilesPerUnit * kPagesPerTile) s.unit_pages[sa][lane] = upage;
            if (lane == 0) {
                s.unit_u[sa] = u_cur;
                s.unit_tiles[sa] = w.ntiles;
                s.unit_nsub[sa] = w.nsub;
            }
            __syncwarp();
            if (lane == 0) {
                // the descriptor is visible to whoever sees either phase complete
                mbar_arrive(&s.desc_full[sa]);
                mbar_arrive_expect_tx(&s.a_full[sa], (uint32_t)w.nsub * 2u * a_box_rows * 128u);
                for (int m = 0; m < w.nsub; ++m) {
                    tc::tma_load_2d(s.a[sa][m][0], &map_q, 0, w.m0 + m * kBM, &s.a_full[sa]);
                    tc::tma_load_2d(s.a[sa][m][1], &map_q, 64, w.m0 + m * kBM, &s.a_full[sa]);
                }
            }
            ++a_fills[sa];
            ++uc;
            if (aborted(s)) break;
        }
        // drain: every buffer this warp filled must have landed before the CTA exits (before the
        // end marker below completes one more phase of a stage)
        if (lane == 0)
            for (int k = 0; k < kStagesA; ++k)
                if (a_fills[k] > 0) mbar_drain(&s.a_full[k], (a_fills[k] - 1) & 1, dev_err);
        __syncwarp();
        // end marker for every other role: a stage that holds no unit
        if (!aborted(s)) {
            const int sa = uc % kStagesA;
            if (warp_wait(&s.a_empty[sa], ((uc / kStagesA) & 1) ^ 1, s, dev_err, lane) && lane == 0) {
                s.unit_tiles[sa] = 0;
                mbar_arrive(&s.desc_full[sa]);
                mbar_arrive(&s.a_full[sa]);
            }
        }
    } else if (warp == kProducerBWarp) {
        // ------------------------------------------------------------ TMA producer: key tiles
        int it = 0, uc = 0;
        int b_fills[kStagesB] = {};
        bool stop = false;
        while (!stop) {
            const int sa = uc % kStagesA;
            if (!warp_wait(&s.desc_full[sa], (uc / kStagesA) & 1, s, dev_err, lane)) break;
            const int ntiles = *(volatile int *)&s.unit_tiles[sa];
            if (ntiles == 0) break;   // end marker
            // lane l < 4 * kTilesPerUnit: block t0 * 4 + l
            const int upage = lane < kTilesPerUnit * kPagesPerTile ? *(volatile int *)&s.unit_pages[sa][lane] : -1;
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.a_empty[sa]);   // descriptor read
            ++uc;
            for (int t = 0; t < ntiles; ++t, ++it) {
                const int st = it % kStagesB;
                int page = __shfl_sync(0xffffffffu, upage, t * kPagesPerTile + (lane & (kPagesPerTile - 1)));
                if (lane >= kPagesPerTile) page = -1;   // lanes 0..3 issue the tile's pages
                const unsigned valid = __ballot_sync(0xffffffffu, page >= 0);
                if (!warp_wait(&s.b_empty[st], ((it / kStagesB) & 1) ^ 1, s, dev_err, lane)) {
                    stop = true;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(&s.b_full[st], (uint32_t)__popc(valid) * 2u * kBoxBytesB);
                __syncwarp();
                if (page >= 0) {   // lane k issues page k's two boxes
                    tc::tma_load_2d(s.b[st][0] + lane * kBoxBytesB, &map_k, 0, page * kBlock, &s.b_full[st]);
                    tc::tma_load_2d(s.b[st][1] + lane * kBoxBytesB, &map_k, 64, page * kBlock, &s.b_full[st]);
                }
                ++b_fills[st];
                if (aborted(s)) {
                    stop = true;
                    break;
                }
            }
        }
        if (lane == 0)
            for (int k = 0; k < kStagesB; ++k)
                if (b_fills[k] > 0) mbar_drain(&s.b_full[k], (b_fills[k] - 1) & 1, dev_err);
    } else if (warp == kMmaWarp || warp == kMmaWarp1) {
        // ------------------------------------------------------------ MMA issuers, one per subtile
        // Two issuing threads: while one waits on a barrier or commits, the other's MMAs keep
        // the tensor pipe busy.  Each stage and accumulator is released by both (count kMT).
        const int m = warp == kMmaWarp ? 0 : 1;
        constexpr uint32_t idesc = tc::idesc_bf16_f32(kBM, kBN);
        static_assert(kTilesPerUnit * kPagesPerTile <= 32, "a unit's page ids fit in one warp");
        static_assert(2 * kMT * kBN == 512, "two accumulator buffers of kMT subtiles fill the 512 TMEM columns");
        static_assert(kMT == 2, "one issuing warp per subtile");
        // the units come from the query producer with their A stages: no unit logic here
        int it = 0, uc = 0;
        bool issued = false, stop = false;
        while (!stop) {
            const int sa = uc % kStagesA;
            if (!warp_wait(&s.a_full[sa], (uc / kStagesA) & 1, s, dev_err, lane)) break;
            const int ntiles = *(volatile int *)&s.unit_tiles[sa];
            const int nsub = *(volatile int *)&s.unit_nsub[sa];
            if (ntiles == 0) break;   // end marker
            ++uc;
            const bool mine = m < nsub;   // this subtile holds queries in the unit
            for (int t = 0; t < ntiles; ++t, ++it) {
                const int st = it % kStagesB;
                const int acc = it & 1;
                if (!warp_wait2(&s.b_full[st], (it / kStagesB) & 1, &s.acc_empty[acc][m], ((it >> 1) & 1) ^ 1, s,
                                dev_err, lane)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    if (mine) {
                        tc::fence_after_sync();
                        // k-step k reads 16 bf16 = 32 bytes further into the 128-byte swizzle row:
                        // 2 more in the descriptor's start-address field (16-byte units; the stage
                        // addresses stay far below the field's 256 KiB range)
                        const uint64_t bd0 = tc::smem_desc_k_sw128(smem_addr(s.b[st][0]));
                        const uint64_t bd1 = tc::smem_desc_k_sw128(smem_addr(s.b[st][1]));
                        const uint64_t ad0 = tc::smem_desc_k_sw128(smem_addr(s.a[sa][m][0]));
                        const uint64_t ad1 = tc::smem_desc_k_sw128(smem_addr(s.a[sa][m][1]));
                        const uint32_t d = tmem + (uint32_t)((acc * kMT + m) * kBN);
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint64_t koff = (uint64_t)((k & 3) * 2);
                            tc::mma_bf16(d, (k < 4 ? ad0 : ad1) + koff, (k < 4 ? bd0 : bd1) + koff, idesc,
                                         k > 0 ? 1u : 0u);
                        }
                        // the epilogue frees the key stage once it sees the accumulator complete
                        tc::commit(&s.acc_full[acc][m]);
                        issued = true;
                    } else {
                        mbar_arrive(&s.acc_full[acc][m]);   // nothing written: at once
                    }
                }
                __syncwarp();
            }
            if (lane == 0) {   // the A subtile is free once its MMAs complete
                if (mine)
                    tc::commit(&s.a_empty[sa]);
                else
                    mbar_arrive(&s.a_empty[sa]);
            }
            __syncwarp();
            if (aborted(s)) break;
        }
        // drain: every MMA this thread issued has completed before TMEM is freed
        if (lane == 0 && issued) {
            tc::commit(&s.mma_done[m]);
            mbar_drain(&s.mma_done[m], 0, dev_err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue, warps 0..7
        const int quarter = warp & 3;            // TMEM lane quarter = rows 32q .. 32q+31 of a subtile
        const int sub = warp >> 2;               // subtile
        int it = 0, uc = 0;
        bool stop = false;
        while (!stop) {
            const int sa = uc % kStagesA;
            if (!warp_wait(&s.desc_full[sa], (uc / kStagesA) & 1, s, dev_err, lane)) break;
            const int ntiles = *(volatile int *)&s.unit_tiles[sa];
            if (ntiles == 0) break;   // end marker
            const int u = *(volatile int *)&s.unit_u[sa];
            const int nsub = *(volatile int *)&s.unit_nsub[sa];
            // which of the unit's blocks have a page in the pool and in the causal range (bit 4t + k)
            const unsigned pool_mask = __ballot_sync(
                0xffffffffu, lane < kTilesPerUnit * kPagesPerTile && *(volatile int *)&s.unit_pages[sa][lane] >= 0);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.a_empty[sa]);   // descriptor read
            ++uc;
            const int m0 = (u / n_chunks) * (kBM * kMT), t0u = (u % n_chunks) * kTilesPerUnit;
            const int row = m0 + sub * kBM + quarter * 32 + lane;
            // the row's position: its load overlaps the wait for the unit's first accumulator
            const int p_raw = row < n_q ? __ldg(q_pos + row) : -1;
            if (row < n_q && p_raw >= seq_len && t0u == 0) flag_error(dev_err, UOCR_DEVERR_POS);
            const int p = (row < n_q && p_raw < seq_len_ok) ? p_raw : -1;
            const int nb_row = p < 0 ? 0 : p / kBlock + 1;
            float *srow = scores + (size_t)(row < n_q ? row : 0) * max_blocks;
            for (int t = 0; t < ntiles; ++t, ++it) {
                const int acc = it & 1;
                if (!warp_wait(&s.acc_full[acc][sub], (it >> 1) & 1, s, dev_err, lane,
                               it == 0 ? first_wait_ns : kWaitLimitNs)) {
                    stop = true;
                    break;
                }
                // this subtile's MMAs of the tile are complete: its reads of the key stage are done
                if (quarter == 0 && lane == 0) mbar_arrive(&s.b_empty[it % kStagesB]);
                tc::fence_after_sync();
                const int tile = t0u + t;
                const int j0 = tile * kPagesPerTile;                     // first block of the tile
                const bool interior = (j0 + 4) * kBlock - 1 <= p;        // no masking needed
                float best[4];
                const uint32_t tbase =
                    tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((acc * kMT + sub) * kBN);
                // a subtile past the last query holds no accumulator: read nothing, write nothing
                const bool have = sub < nsub;
                if (have) {
                    // the tile's 4 blocks in one TMEM round trip (4 x 32 columns in flight)
                    float v[4][32];
#pragma unroll
                    for (int k = 0; k < 4; ++k) tc::tmem_ld_32x32b_x32(tbase + k * 32, v[k]);
                    tc::tmem_ld_wait();
                    if (interior) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
#pragma unroll
                            for (int c = 16; c > 0; c >>= 1)
#pragma unroll
                                for (int x = 0; x < c; ++x) v[k][x] = fmaxf(v[k][x], v[k][x + c]);
                            best[k] = v[k][0];
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int t0 = (j0 + k) * kBlock;
                            float m = -INFINITY;
#pragma unroll
                            for (int c = 0; c < 32; ++c) m = (t0 + c <= p) ? fmaxf(m, v[k][c]) : m;
                            best[k] = m;
                        }
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&s.acc_empty[acc][sub]);
                if (!have) continue;
                // a block whose page is not in the pool scores -inf; blocks past the row's
                // causal range are not written
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (!((pool_mask >> (t * kPagesPerTile + k)) & 1u)) best[k] = -INFINITY;
                if (j0 + 4 <= nb_row && (reinterpret_cast<uintptr_t>(srow + j0) & 15u) == 0) {
                    *reinterpret_cast<float4 *>(srow + j0) = make_float4(best[0], best[1], best[2], best[3]);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (j0 + k < nb_row) srow[j0 + k] = best[k];
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side
EncodeTiledFn tensor_map_encoder() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
}

namespace {

// 2-D bf16 tensor of `rows` x 128 (row stride 256 B), boxes of 64 x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {128, rows};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_index_gemm_smem() { return sizeof(Smem) + 1024; }

cudaError_t launch_prefill_index_gemm(const LaunchCtx &c, const void *idx_q, const void *idx_k,
                                      const int32_t *bt_row, const int32_t *seq_len_ptr, const int32_t *q_pos,
                                      int n_q, int max_blocks, int num_pages, float *scores, int32_t *sched,
                                      int32_t *dev_err) {
    const int a_box_rows = n_q < kBM ? n_q : kBM;
    CUtensorMap map_q, map_k;
    if (!make_map(&map_q, idx_q, (uint64_t)n_q, (uint32_t)a_box_rows)) return cudaErrorInvalidValue;
    if (!make_map(&map_k, idx_k, (uint64_t)num_pages * kBlock, kBlock)) return cudaErrorInvalidValue;
    const int m_tiles = (n_q + kBM * kMT - 1) / (kBM * kMT);
    const int n_tiles = (max_blocks + kPagesPerTile - 1) / kPagesPerTile;
    const int n_chunks = (n_tiles + kTilesPerUnit - 1) / kTilesPerUnit;
    const long long units = (long long)m_tiles * n_chunks;
    if (units > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const int grid = (int)(units < c.num_sms ? units : c.num_sms);
    const size_t smem = prefill_index_gemm_smem();
    cudaError_t e = cudaFuncSetAttribute(prefill_index_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, prefill_index_gemm_kernel, map_q, map_k, bt_row, seq_len_ptr, q_pos, n_q,
                              a_box_rows, num_pages, max_blocks, n_chunks, (int)units, scores, sched, dev_err,
                              c.first_wait_ns);
}

}  // namespace uocr
