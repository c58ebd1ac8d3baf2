// kernels.h -- internal launchers of libuocr (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "uocr.h"

namespace uocr {

struct LaunchCtx {
    cudaStream_t stream;
    int num_sms;
    bool pdl;   // launch with programmatic stream serialization
    // Limit of the first bounded wait of the decode attention (its V copy) and of the scoring
    // GEMM's epilogue (its first accumulator); kWaitLimitNs except when a test shortens it to
    // exercise the timeout path.  Every other wait keeps kWaitLimitNs.
    uint64_t first_wait_ns;
};

cudaError_t launch_index_scan(const LaunchCtx &c, const void *idx_q, const void *idx_k,
                              const int32_t *bt, const int32_t *seq_lens, const int32_t *q_seq,
                              const int32_t *q_pos, int n_q, int B, int max_blocks, int num_pages,
                              float *scores, int32_t *dev_err);

cudaError_t launch_block_topk(const LaunchCtx &c, const float *scores, const int32_t *seq_lens,
                              const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                              int max_blocks, int32_t *sel, int32_t *dev_err, int fixed_seq = -1,
                              const uint32_t *cand_mask = nullptr, int mask_words = 0,
                              int32_t *counts = nullptr);

cudaError_t launch_sparse_attn(const LaunchCtx &c, const void *q, const void *k, const void *v,
                               const int32_t *bt, const int32_t *seq_lens, const int32_t *q_seq,
                               const int32_t *q_pos, const int32_t *sel, int n_q, int B, int H,
                               int max_blocks, int num_pages, float scale, void *out,
                               bool implicit_local, int fixed_seq, bool head_major, int32_t *dev_err);

// The argument checks of uocr_sparse_decode other than the workspace's (shared with
// uocr_sparse_decode_static, which checks its fixed scratch size after them).
uocr_status_t check_sparse_decode_args(const void *q, const void *k_cache, const void *v_cache, const void *idx_q,
                                       const void *idx_k_cache, const int32_t *block_table,
                                       const int32_t *seq_lens, int B, int H, int max_blocks, int num_pages,
                                       const void *out, const int32_t *sel_out, const int32_t *dev_err);

// tcgen05 block scoring of n_q queries of one sequence (block table row bt_row,
// length *seq_len_ptr) into scores [n_q][max_blocks].  sched: a zeroed int32 work-unit counter
// for this launch alone (CTAs take units as they go), or NULL for a round-robin split.
cudaError_t launch_prefill_index_gemm(const LaunchCtx &c, const void *idx_q, const void *idx_k,
                                      const int32_t *bt_row, const int32_t *seq_len_ptr, const int32_t *q_pos,
                                      int n_q, int max_blocks, int num_pages, float *scores, int32_t *sched,
                                      int32_t *dev_err);

// cuTensorMapEncodeTiled through the runtime's driver entry point (NULL if unavailable).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Prefill attention of many queries of one sequence over their selection: the selection is
// classified per 128-query tile (local-window entries of tiles whose windows fit 8 blocks go to
// the tensor-core local kernel, the rest to the block kernel), the block kernel's entries are
// inverted per block and attended in items of 16 entries per (block, head), and a merge kernel
// combines each row's partial states.  Workspace regions, 256-byte aligned.  The first zero_bytes
// bytes (per-block entry counts, list counters, the scoring GEMM's and the block kernel's unit
// counters) must be zero before the call's first kernel.
struct PrefillAttnWs {
    size_t counts_off, fill_off, sched_off, blk_sched_off, n_items_off, items_off, list_off, sel_off, loc_off,
        tile_off, ml_off, o_off, loc_ml_off, loc_o_off;
    size_t zero_bytes;
};
size_t prefill_attn_workspace(int n_q, int H, int max_blocks, PrefillAttnWs *w);
// sel: the queries' selection ([n_q][16], any order, -1 for an empty slot), validated here.
cudaError_t launch_prefill_attn(const LaunchCtx &c, const void *q, const void *k, const void *v,
                                const int32_t *bt_row, const int32_t *seq_len_ptr, const int32_t *q_pos,
                                const int32_t *sel, int n_q, int H, int max_blocks, int num_pages, float scale,
                                void *out, void *ws, int32_t *dev_err);
// The kernels of prefill_local.cu (launched by launch_prefill_attn).
int prefill_local_tiles(int n_q);
// TMA map of a K or V cache [P][H][32][128] bf16 as a 3-D tensor (dim, token, page * H + head)
// read in boxes of 64 dims x 32 tokens with the 128-byte swizzle.
bool prefill_kv_tensor_map(CUtensorMap *map, const void *cache, int num_pages, int H);
cudaError_t launch_prefill_classify(const LaunchCtx &c, const int32_t *sel, const int32_t *q_pos,
                                    const int32_t *seq_len_ptr, int n_q, int max_blocks, int32_t *sel_ws,
                                    int32_t *counts, int32_t *loc_info, int2 *tile_info, int32_t *dev_err);
cudaError_t launch_prefill_local(const LaunchCtx &c, const void *q, const void *k, const void *v,
                                 const int32_t *bt_row, const int32_t *q_pos, const int32_t *loc_info,
                                 const int2 *tile_info, int n_q, int H, int num_pages, float scale, void *loc_o,
                                 float2 *loc_ml, int32_t *dev_err);
cudaError_t launch_prefill_merge(const LaunchCtx &c, const int32_t *sel_ws, const void *part_o, const float *part_ml,
                                 const void *loc_o, const float2 *loc_ml, int n_q, int H, void *out);

// Comparator decode attention over [0, min(ref_blocks, nb)) U the 4-block local window.
int dense_chunks(int max_blocks);
size_t dense_attn_workspace(int n_q, int H, int max_blocks);
cudaError_t launch_dense_attn(const LaunchCtx &c, const void *q, const void *k, const void *v, const int32_t *bt,
                              const int32_t *seq_lens, int B, int H, int max_blocks, int num_pages, int ref_blocks,
                              float scale, void *out, void *ws, int32_t *dev_err);

// page2d rotary embedding + cache append of new tokens.
struct RopeFreqs {
    double inv[UOCR_HEAD_DIM / 2];   // per frequency pair: radians per unit of its coordinate
};
RopeFreqs rope_freqs();
cudaError_t launch_rope_append(const LaunchCtx &c, void *q, void *idx_q, const void *k_new, const void *v_new,
                               const void *idx_k_new, const int32_t *tok_pos, const int32_t *page_pos,
                               const int32_t *q_seq, const int32_t *q_pos, const int32_t *bt,
                               const int32_t *seq_lens, int n, int B, int H, int max_blocks, int num_pages,
                               void *k_cache, void *v_cache, void *idx_k_cache, int32_t *dev_err);

// Block-summary scoring (one summary vector per page) and the mean-key summary builder.
cudaError_t launch_summary_scan(const LaunchCtx &c, const void *idx_q, const void *summary, const int32_t *bt,
                                const int32_t *seq_lens, const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                                int max_blocks, int num_pages, float *scores, int32_t *dev_err);
cudaError_t launch_block_mean(const LaunchCtx &c, const void *idx_k, const int32_t *pages, int n_pages,
                              int num_pages, void *summary, int32_t *dev_err);

}  // namespace uocr
