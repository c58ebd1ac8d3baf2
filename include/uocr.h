/*
 * uocr.h -- C ABI of libuocr.so: the SR-SWA / DASH block-sparse attention step
 * of Unlimited-OCR-2 on NVIDIA B200 (sm_100a).
 *
 * What the step computes (cited by page and section):
 *   [rkmt]  Unlimited-OCR-2 walk-through, news.rkmt.cn/news/25027, section 五
 *           ("SR-SWA: block-level sparse attention"): keys are cut into 32-token
 *           blocks (step 1); a 1-head x 128-dim Lightning Indexer scores every
 *           block for every query, the block score being the maximum over the
 *           block's tokens (step 2); each query keeps 16 blocks, 4 local blocks
 *           (the 128-token sliding window) plus 12 remote blocks (step 3); exact
 *           attention runs over the selected blocks only (step 4).  Section 三:
 *           10 attention heads, 10 KV heads (MHA), head dim 128.
 *   [lqnn]  Unlimited-OCR-2-8bit page, www.lqnn.cn/news/271890, section
 *           显存账本: top-12 remote + 4 local = 16 blocks x 32 = 512 tokens.
 *   [leheaven] release report, leheavengame.com (Unlimited OCR 2 open-source),
 *           section 三: chunked prefill materialises a [tokens, context/32]
 *           block-score tensor.
 *
 * Readings where the pages are open (the same in the CPU oracle):
 *   - block score = max over tokens t <= p of the raw dot product q_idx . k_idx
 *     (no ReLU, no weight, no scale);
 *   - a query at position p sees tokens 0..p; nb = p/32 + 1 causal blocks;
 *     local = the last 4 causal blocks, remote candidates = blocks [0, nb-4);
 *   - remote ranking: score descending, then lower block id; with no more than
 *     12 candidates all of them are taken;
 *   - the decode query is the last cached token: p = seq_len - 1.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates or frees device memory and, apart from the one fixed
 *     scratch array of uocr_sparse_decode_static (see its declaration), keeps
 *     no device memory and no global state.
 *   - bf16 tensors are passed as void* (IEEE bfloat16 bit patterns), must be
 *     16-byte aligned and densely packed in the layouts given below.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default stream)
 *     and performs no host/device synchronisation.
 *   - Host-side argument checks run before any launch; a failed check returns
 *     UOCR_ERR_INVALID_ARG / UOCR_ERR_UNSUPPORTED / UOCR_ERR_WORKSPACE and
 *     launches nothing.  A failed launch returns UOCR_ERR_CUDA.
 *   - Data-dependent checks run on the device: a block-table entry outside
 *     [0, num_pages), a query position at or past its sequence length, a
 *     sequence index outside [0, B), or more causal blocks than max_blocks make
 *     the kernel skip the offending block / query (its outputs are -inf scores,
 *     -1 selections, zero attention output) and, when `dev_err` is not NULL,
 *     OR a UOCR_DEVERR_* bit into *dev_err.  Kernels never trap.
 *
 * Layouts (P = num_pages, B = sequences, n_q = queries, H = heads):
 *   q            bf16  [n_q][H][128]
 *   k_cache      bf16  [P][H][32][128]   one (page, head) tile = 8 KiB contiguous
 *   v_cache      bf16  [P][H][32][128]
 *   idx_q        bf16  [n_q][128]
 *   idx_k_cache  bf16  [P][32][128]      one page = 8 KiB contiguous
 *   block_table  int32 [B][max_blocks]   logical block j of sequence b -> page
 *   seq_lens     int32 [B]               cached tokens of each sequence
 *   q_seq        int32 [n_q]             sequence of each query (NULL: query i -> sequence i)
 *   q_pos        int32 [n_q]             token position p of each query (NULL: seq_len - 1)
 *   scores       fp32  [n_q][max_blocks] block scores; entries j >= nb are not written
 *   sel          int32 [n_q][16]         selected logical blocks, ascending, -1 padded
 *   out          bf16  [n_q][H][128]
 */
#ifndef UOCR_H
#define UOCR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t / CUstream. */
typedef struct CUstream_st *uocr_stream_t;

typedef enum {
    UOCR_OK = 0,
    UOCR_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, misaligned pointer */
    UOCR_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement */
    UOCR_ERR_WORKSPACE = 3,     /* workspace NULL, misaligned or too small */
    UOCR_ERR_CUDA = 4           /* a CUDA launch or attribute call failed */
} uocr_status_t;

/* Method constants ([rkmt 五], [lqnn 显存账本]). */
#define UOCR_BLOCK 32
#define UOCR_N_LOCAL 4
#define UOCR_N_REMOTE 12
#define UOCR_N_SEL 16
#define UOCR_HEAD_DIM 128
#define UOCR_IDX_DIM 128
#define UOCR_MAX_HEADS 64
/* page2d rotary embedding ([rkmt 四], [rkmt 六]). */
#define UOCR_ROPE_PAGE_PAIRS 1      /* frequency pairs on the page axis (of 64) */
#define UOCR_ROPE_PAGE_MOD 2        /* page coordinate = page % 2 */
#define UOCR_ROPE_THETA_TOKEN 10000.0
#define UOCR_ROPE_THETA_PAGE 256.0

/* Bits OR-ed into *dev_err by the kernels. */
#define UOCR_DEVERR_PAGE 1u   /* block-table entry outside [0, num_pages) */
#define UOCR_DEVERR_POS 2u    /* q_pos >= seq_len, q_seq outside [0, B), or nb > max_blocks */
#define UOCR_DEVERR_SEL 4u    /* a selected block outside the query's causal blocks */
#define UOCR_DEVERR_TIMEOUT 8u /* a bounded wait on an asynchronous copy gave up (block skipped) */

/* Human-readable name of a status code (static storage; never NULL). */
const char *uocr_status_string(uocr_status_t status);

/* ABI version of this header; bumped on any signature change. */
int uocr_abi_version(void);

/*
 * The CUDA runtime's description of the error behind the calling thread's
 * most recent UOCR_ERR_CUDA ("no error" if there was none): which launch or
 * attribute call failed and why.  Static storage; never NULL.
 */
const char *uocr_last_cuda_error(void);

/*
 * Workspace bytes that uocr_sparse_decode and uocr_sparse_prefill need for n_q queries over
 * max_blocks blocks: the fp32 block scores [n_q][max_blocks], rounded up to
 * 256 bytes.  A pure function of the shapes (0 for a non-positive argument);
 * H is accepted for symmetry with the other entry points and does not change
 * the result.  Callers may reuse one workspace across calls on one stream.
 */
size_t uocr_workspace_bytes(int n_q, int H, int max_blocks);

/*
 * Indexer scan, [rkmt 五 steps 1-2]:
 *   scores[i][j] = max_{t in block j, t <= p_i} sum_{d<128} idx_q[i][d] * idx_k[t][d]
 * for every causal block j < nb_i of query i, in fp32 from bf16 inputs.
 * HBM-bound: reads every causal indexer page of the query's sequence once.
 * Errors: INVALID_ARG for NULL idx_q / idx_k_cache / block_table / seq_lens /
 * scores, n_q < 0, B < 1, max_blocks < 1, num_pages < 1, or misalignment.
 */
uocr_status_t uocr_index_score(const void *idx_q, const void *idx_k_cache,
                               const int32_t *block_table, const int32_t *seq_lens,
                               const int32_t *q_seq, const int32_t *q_pos,
                               int n_q, int B, int max_blocks, int num_pages,
                               float *scores, int32_t *dev_err, uocr_stream_t stream);

/*
 * Block selection, [rkmt 五 step 3]: for each query, the local blocks
 * {nb-4, ..., nb-1} (clipped at 0) and the 12 highest-scoring remote
 * candidates in [0, nb-4), ranked by (score desc, block id asc); all
 * candidates when there are at most 12.  sel[i] = the union, ascending, -1
 * padded to 16.  Reads scores[i][0 .. nb-5] only.
 */
uocr_status_t uocr_block_topk(const float *scores, const int32_t *seq_lens,
                              const int32_t *q_seq, const int32_t *q_pos,
                              int n_q, int B, int max_blocks, int32_t *sel,
                              int32_t *dev_err, uocr_stream_t stream);

/*
 * Gathered exact attention, [rkmt 五 step 4]: per query i and head h,
 *   z_t = scale * q[i][h] . k[h][t]  over the tokens t <= p_i of the blocks in sel[i],
 *   out[i][h] = sum_t softmax(z)_t v[h][t]    (fp32 softmax and accumulation, bf16 out).
 * Entries of sel < 0 are skipped; a query with no visible token gets zeros.
 * Split-K over the 16 blocks (one thread-block cluster of 4 CTAs per query
 * and head) with the flash-decoding merge done on chip: no workspace.
 * H in [1, UOCR_MAX_HEADS] (the model uses 10); head dim fixed at 128.
 */
uocr_status_t uocr_sparse_attn(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_table, const int32_t *seq_lens,
                               const int32_t *q_seq, const int32_t *q_pos,
                               const int32_t *sel, int n_q, int B, int H,
                               int max_blocks, int num_pages, float scale, void *out,
                               int32_t *dev_err, uocr_stream_t stream);

/*
 * The whole decode step for B sequences, one query each at p = seq_len - 1:
 * uocr_index_score -> uocr_block_topk -> uocr_sparse_attn with
 * scale = 1/sqrt(128), launched back to back on `stream` (programmatic
 * dependent launch, no host synchronisation).  sel_out [B][16] receives the
 * selection and must not be NULL.  Workspace: uocr_workspace_bytes(B, H, max_blocks).
 */
uocr_status_t uocr_sparse_decode(const void *q, const void *k_cache, const void *v_cache,
                                 const void *idx_q, const void *idx_k_cache,
                                 const int32_t *block_table, const int32_t *seq_lens,
                                 int B, int H, int max_blocks, int num_pages,
                                 void *out, int32_t *sel_out,
                                 void *workspace, size_t workspace_bytes,
                                 int32_t *dev_err, uocr_stream_t stream);

/*
 * Chunked-prefill block scores on the tensor cores, [leheaven 三] with the
 * scoring rule of [rkmt 五 step 2]: the same scores as uocr_index_score for
 * n_q queries that all belong to sequence `seq`, at positions q_pos[i]
 * (required; a position at or past seq_lens[seq] flags UOCR_DEVERR_POS and
 * scores nothing), computed as S = idx_q . idx_k^T on tcgen05 (bf16 inputs,
 * fp32 accumulation in TMEM) with the causal mask and the per-block maximum
 * applied while the accumulator is read back.  scores [n_q][max_blocks];
 * entries j >= nb_i are not written.  Needs an sm_100a device; one persistent
 * CTA per SM holds ~193 KiB of shared memory and 512 TMEM columns.
 */
uocr_status_t uocr_prefill_index_score(const void *idx_q, const void *idx_k_cache,
                                       const int32_t *block_table, const int32_t *seq_lens,
                                       int seq, const int32_t *q_pos, int n_q, int B,
                                       int max_blocks, int num_pages, float *scores,
                                       int32_t *dev_err, uocr_stream_t stream);

/*
 * Exact attention of n_q queries of one sequence `seq` over the blocks a
 * caller selected for them: the result of uocr_sparse_attn with q_seq all
 * `seq`, computed block-centrically for many queries (the attention of
 * uocr_sparse_prefill).  [rkmt 五 step 4]
 *   q        [n_q][H][128] bf16 (device)
 *   q_pos    [n_q] int32 positions, required; sel [n_q][16] int32 block ids
 *            (-1 = empty slot), in any order
 *   out      [n_q][H][128] bf16 (device)
 * A slot naming a block that is not causal for its query (id >= p / 32 + 1)
 * is ignored and sets UOCR_DEVERR_SEL; a query at a position outside
 * [0, seq_len) gets a zero output and sets UOCR_DEVERR_POS; a block whose page
 * is outside the pool contributes nothing and sets UOCR_DEVERR_PAGE.  The
 * per-slot partial outputs are rounded to bf16 before the merge (at most
 * 2^-9 max|v| on an output), and the tensor-core products take the softmax
 * weights in bf16.  Workspace: uocr_sparse_attn_seq_workspace_bytes
 * bytes, 256-byte aligned, owned by the caller, a pure function of the shapes.
 * After the call its partial region holds undefined bytes: the merge drops the
 * partials' L2 lines once it has read them, without writing them back.
 */
size_t uocr_sparse_attn_seq_workspace_bytes(int n_q, int H, int max_blocks);

uocr_status_t uocr_sparse_attn_seq(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_table, const int32_t *seq_lens, int seq,
                                   const int32_t *q_pos, const int32_t *sel, int n_q, int B, int H,
                                   int max_blocks, int num_pages, float scale, void *out,
                                   void *workspace, size_t workspace_bytes,
                                   int32_t *dev_err, uocr_stream_t stream);

/*
 * The whole chunked-prefill step for n_q queries of sequence `seq` at
 * positions q_pos (their K/V and indexer keys already cached), launched back
 * to back on `stream`: block scores on the tensor cores (as
 * uocr_prefill_index_score), the selection (as uocr_block_topk: each query
 * keeps its own 4 local + 12 remote blocks over its causal prefix), and exact
 * attention over the selected blocks with scale = 1/sqrt(128) (the result of
 * uocr_sparse_attn).  out [n_q][H][128] bf16, sel_out [n_q][16] int32.
 * The local windows of a tile of 128 consecutive queries share one window of
 * at most 8 blocks and are attended per (tile, head) on the tensor cores
 * (tcgen05, one partial per query and head); the other selected blocks are
 * attended block-centrically: the selection is inverted per block, every
 * selected (block, head) K/V tile is read once for all the queries that chose
 * it, and each (query, slot, head) partial -- the row maximum and weight sum in
 * fp32, the unnormalised partial output in bf16 -- is merged per (query, head).
 * The softmax weights are rounded to bf16 for the tensor-core products (the
 * weight sums add the rounded weights), and the bf16 partials add at most
 * 2^-9 max|v| to an output, the size of the output's own bf16 rounding.  Workspace: uocr_prefill_workspace_bytes(n_q, H,
 * max_blocks) bytes, 256-byte aligned (the block scores first, then the
 * inverted index and the partials; after the call the block scores are
 * readable and the partial region holds undefined bytes, dropped from L2 by
 * the merge without being written back).  Errors as uocr_sparse_decode; a selected
 * block whose page is outside the pool contributes nothing to the output and
 * sets UOCR_DEVERR_PAGE.
 */
/* Workspace bytes uocr_sparse_prefill needs; a pure function of the shapes. */
size_t uocr_prefill_workspace_bytes(int n_q, int H, int max_blocks);

uocr_status_t uocr_sparse_prefill(const void *q, const void *k_cache, const void *v_cache,
                                  const void *idx_q, const void *idx_k_cache,
                                  const int32_t *block_table, const int32_t *seq_lens,
                                  int seq, const int32_t *q_pos, int n_q, int B, int H,
                                  int max_blocks, int num_pages, void *out, int32_t *sel_out,
                                  void *workspace, size_t workspace_bytes,
                                  int32_t *dev_err, uocr_stream_t stream);

/*
 * page2d rotary embedding + cache append for n new tokens, the step before the
 * indexer scan of a decode call ([rkmt 四 page2d], [rkmt 六]).  Token i has
 * in-page offset tok_pos[i] and page number page_pos[i]; of the 64 frequency
 * pairs of a 128-dim head, pairs 0..62 rotate by tok * 10000^(-i/63) and pair 63
 * by (page % 2) * 256^0, rotate-half layout (pair i = dims i and i + 64).
 *   q [n][H][128], idx_q [n][128]      rotated in place;
 *   k_new, v_new [n][H][128], idx_k_new [n][128]
 *                                      rotated k / idx_k and raw v are written to
 *                                      row p % 32 of page block_table[b][p / 32]
 *                                      of k_cache, idx_k_cache and v_cache,
 * for token i of sequence b = q_seq[i] (NULL: i) at position p = q_pos[i]
 * (NULL: seq_lens[b] - 1, i.e. seq_lens already counts the new token).
 * Angles are formed in fp64 and reduced before an fp32 sincos; outputs are
 * rounded to bf16.  Two new tokens must not target the same cache row.
 */
uocr_status_t uocr_rope_append(void *q, void *idx_q, const void *k_new, const void *v_new,
                               const void *idx_k_new, const int32_t *tok_pos, const int32_t *page_pos,
                               const int32_t *q_seq, const int32_t *q_pos,
                               const int32_t *block_table, const int32_t *seq_lens,
                               int n, int B, int H, int max_blocks, int num_pages,
                               void *k_cache, void *v_cache, void *idx_k_cache,
                               int32_t *dev_err, uocr_stream_t stream);

/*
 * Block-summary scoring ([lqnn 显存账本]: "learnable summary vectors" per KV
 * block; [leheaven 二] Token Sieve: score each block by its brief
 * representation, then read the chosen blocks' tokens).  For every causal block
 * j < nb_i of query i:  scores[i][j] = idx_q[i] . summary_cache[block_table[b][j]]
 * with summary_cache bf16 [P][128] (one vector per page, supplied by the caller
 * or built by uocr_block_summary_mean).  32x fewer bytes than the max-over-tokens
 * scan.  Same arguments, layouts and errors as uocr_index_score otherwise.
 */
uocr_status_t uocr_summary_score(const void *idx_q, const void *summary_cache,
                                 const int32_t *block_table, const int32_t *seq_lens,
                                 const int32_t *q_seq, const int32_t *q_pos,
                                 int n_q, int B, int max_blocks, int num_pages,
                                 float *scores, int32_t *dev_err, uocr_stream_t stream);

/*
 * summary_cache[page] = bf16(mean of the page's 32 indexer keys) for the
 * n_pages pages listed in `pages` (NULL: pages 0 .. n_pages-1).  The mean is the
 * summary that needs no trained weights.  summary_cache bf16 [num_pages][128].
 */
uocr_status_t uocr_block_summary_mean(const void *idx_k_cache, const int32_t *pages, int n_pages,
                                      int num_pages, void *summary_cache, int32_t *dev_err,
                                      uocr_stream_t stream);

/*
 * uocr_sparse_decode with block-summary scoring: uocr_summary_score ->
 * uocr_block_topk -> uocr_sparse_attn, same arguments except summary_cache
 * [P][128] in place of the indexer key cache.
 */
uocr_status_t uocr_sparse_decode_summary(const void *q, const void *k_cache, const void *v_cache,
                                         const void *idx_q, const void *summary_cache,
                                         const int32_t *block_table, const int32_t *seq_lens,
                                         int B, int H, int max_blocks, int num_pages,
                                         void *out, int32_t *sel_out,
                                         void *workspace, size_t workspace_bytes,
                                         int32_t *dev_err, uocr_stream_t stream);

/*
 * Block selection under a page-aware candidate constraint ([rkmt 五]
 * image_bucket_constraint: candidates restricted to the current page's image
 * blocks + the local window + a global fallback).  As uocr_block_topk, but a
 * remote candidate j of a query of sequence b may be picked only if bit
 * (cand_mask[b * mask_words + j / 32] >> (j % 32)) & 1 is set; the local window
 * is kept regardless.  With at most 12 allowed candidates all of them are
 * taken; sel is ascending and -1 padded.  mask_words >= ceil(max_blocks / 32).
 */
uocr_status_t uocr_block_topk_masked(const float *scores, const int32_t *seq_lens,
                                     const int32_t *q_seq, const int32_t *q_pos,
                                     const uint32_t *cand_mask, int mask_words,
                                     int n_q, int B, int max_blocks, int32_t *sel,
                                     int32_t *dev_err, uocr_stream_t stream);

/*
 * Comparator decode attention (baselines the pages quote the sparse step
 * against: full attention and R-SWA; release report, leheavengame.com, section
 * 一: 7.0x and 5.6x; R-SWA: Unlimited OCR v1 article, chenxutan.com/d/4261.html,
 * section 2.3.2).  For each sequence's decode query (p = seq_len - 1), exact
 * softmax attention (scale 1/sqrt(128)) over the tokens t <= p of the blocks
 *   [0, min(ref_blocks, nb))  U  [max(nb - 4, 0), nb)
 * i.e. a reference prefix plus the 128-token local window; ref_blocks >=
 * max_blocks gives full causal attention.  Split-K over 16-block chunks with a
 * merge kernel.  Workspace: uocr_dense_workspace_bytes(B, H, max_blocks).
 */
size_t uocr_dense_workspace_bytes(int B, int H, int max_blocks);
uocr_status_t uocr_dense_decode(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_table, const int32_t *seq_lens, int ref_blocks,
                                int B, int H, int max_blocks, int num_pages, void *out,
                                void *workspace, size_t workspace_bytes, int32_t *dev_err,
                                uocr_stream_t stream);

/*
 * uocr_sparse_decode_static -- uocr_sparse_decode for callers that cannot
 * allocate device memory (for example a plugin inside a host engine that owns
 * every device allocation, or a decode loop where a cudaMalloc, which may
 * synchronise the device, is not allowed).  The paper has no counterpart: this
 * is a packaging variant, not a step of the method.
 *
 * Same arguments, layouts, checks and results as uocr_sparse_decode, without
 * the workspace: the scratch lives in one device array of
 * UOCR_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library keeps until the process exits.  Nothing is allocated or freed.
 *   - Returns UOCR_ERR_WORKSPACE, launching nothing, when
 *     uocr_workspace_bytes(B, H, max_blocks) > UOCR_STATIC_SCRATCH_BYTES
 *     (e.g. B = 64 sequences fit up to max_blocks = 32768, 1M tokens each).
 *   - The first call on a device (with that device current) looks up the
 *     array's device address and caches it; make that first call before any
 *     stream capture on that device.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents (no part of it needs to start at zero).  Calls whose kernels
 *     overlap on the GPU -- several streams, or several host threads -- race
 *     on it: serialise them.
 */
#define UOCR_STATIC_SCRATCH_BYTES (8u << 20)

uocr_status_t uocr_sparse_decode_static(const void *q, const void *k_cache, const void *v_cache,
                                        const void *idx_q, const void *idx_k_cache,
                                        const int32_t *block_table, const int32_t *seq_lens,
                                        int B, int H, int max_blocks, int num_pages,
                                        void *out, int32_t *sel_out,
                                        int32_t *dev_err, uocr_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* UOCR_H */
