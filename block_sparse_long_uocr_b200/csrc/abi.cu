// abi.cu -- the extern "C" entry points of libuocr.so (declared in include/uocr.h).
//
// Host side only: argument validation, workspace carving, device attribute
// lookup and the launches on the caller's stream.  No allocation, no
// synchronisation, no state kept between calls.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "uocr.h"

namespace {

constexpr size_t kWsAlign = 256;

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

struct WsLayout {
    size_t scores_off, total;
};

// The workspace holds the block scores [n_q][max_blocks] f32 (the attention merges its
// split-K partials on chip, so it needs none).
inline WsLayout ws_layout(int n_q, int /*H*/, int max_blocks) {
    WsLayout w{};
    w.scores_off = 0;
    w.total = round_up((size_t)n_q * max_blocks * sizeof(float), kWsAlign);
    return w;
}

// The CUDA error behind this thread's last UOCR_ERR_CUDA (uocr_last_cuda_error).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

inline uocr_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return UOCR_OK;
    t_last_cuda_error = e;
    (void)cudaGetLastError();   // clear the sticky-free launch error so later calls are clean
    return UOCR_ERR_CUDA;
}

// Limit of the first bounded wait of the decode attention and of the scoring GEMM's epilogue
// (LaunchCtx::first_wait_ns), negative for the library default.  Set only by the test hook
// uocr_test_first_wait_limit_ns below.
std::atomic<long long> g_first_wait_ns{-1};

inline uocr_status_t make_ctx(uocr_stream_t stream, bool pdl, uocr::LaunchCtx &c) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_status(e);
    c.stream = (cudaStream_t)stream;
    c.num_sms = sms;
    c.pdl = pdl;
    const long long w = g_first_wait_ns.load(std::memory_order_relaxed);
    c.first_wait_ns = w < 0 ? uocr::kWaitLimitNs : (uint64_t)w;
    return UOCR_OK;
}

// Common shape checks shared by every compute entry point.
inline uocr_status_t check_common(int n_q, int B, int max_blocks, int num_pages,
                                  const int32_t *block_table, const int32_t *seq_lens,
                                  const int32_t *q_seq, const int32_t *q_pos, const int32_t *dev_err) {
    if (n_q < 0 || B < 1 || max_blocks < 1 || num_pages < 1) return UOCR_ERR_INVALID_ARG;
    if (!block_table || !seq_lens) return UOCR_ERR_INVALID_ARG;
    if (!aligned(block_table, 4) || !aligned(seq_lens, 4)) return UOCR_ERR_INVALID_ARG;
    if ((q_seq && !aligned(q_seq, 4)) || (q_pos && !aligned(q_pos, 4))) return UOCR_ERR_INVALID_ARG;
    if (dev_err && !aligned(dev_err, 4)) return UOCR_ERR_INVALID_ARG;
    if ((long long)max_blocks * UOCR_BLOCK > 0x7fffffffLL) return UOCR_ERR_UNSUPPORTED;
    return UOCR_OK;
}

inline bool bf16_ok(const void *p) { return p && aligned(p, 16); }

}  // namespace

extern "C" {

const char *uocr_status_string(uocr_status_t status) {
    switch (status) {
        case UOCR_OK: return "UOCR_OK";
        case UOCR_ERR_INVALID_ARG: return "UOCR_ERR_INVALID_ARG: NULL pointer, bad size or misaligned pointer";
        case UOCR_ERR_UNSUPPORTED: return "UOCR_ERR_UNSUPPORTED: shape outside what the kernels implement";
        case UOCR_ERR_WORKSPACE: return "UOCR_ERR_WORKSPACE: workspace NULL, misaligned or too small";
        case UOCR_ERR_CUDA: return "UOCR_ERR_CUDA: a CUDA launch or attribute query failed";
    }
    return "UOCR_ERR_UNKNOWN";
}

int uocr_abi_version(void) { return 2; }

const char *uocr_last_cuda_error(void) {
    return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

// Test hook, not part of the ABI in uocr.h: sets the wall-time limit of the first bounded wait
// of the decode attention (its V copy) and of the scoring GEMM's epilogue (its first
// accumulator) for the calls that follow, process-wide; ns = 0 makes those waits give up at
// once, a negative ns restores the default (2 s).  The drain waits that follow a timeout keep
// the default limit.  Used by the tests to run the timeout paths without a stuck copy.
void uocr_test_first_wait_limit_ns(long long ns) { g_first_wait_ns.store(ns, std::memory_order_relaxed); }

size_t uocr_workspace_bytes(int n_q, int H, int max_blocks) {
    if (n_q <= 0 || H <= 0 || max_blocks <= 0) return 0;
    return ws_layout(n_q, H, max_blocks).total;
}

uocr_status_t uocr_index_score(const void *idx_q, const void *idx_k_cache,
                               const int32_t *block_table, const int32_t *seq_lens,
                               const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                               int max_blocks, int num_pages, float *scores, int32_t *dev_err,
                               uocr_stream_t stream) {
    uocr_status_t st = check_common(n_q, B, max_blocks, num_pages, block_table, seq_lens, q_seq,
                                    q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(idx_q) || !bf16_ok(idx_k_cache) || !scores || !aligned(scores, 4))
        return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_index_scan(c, idx_q, idx_k_cache, block_table, seq_lens, q_seq,
                                               q_pos, n_q, B, max_blocks, num_pages, scores, dev_err));
}

uocr_status_t uocr_block_topk(const float *scores, const int32_t *seq_lens, const int32_t *q_seq,
                              const int32_t *q_pos, int n_q, int B, int max_blocks, int32_t *sel,
                              int32_t *dev_err, uocr_stream_t stream) {
    if (n_q < 0 || B < 1 || max_blocks < 1) return UOCR_ERR_INVALID_ARG;
    if (!scores || !seq_lens || !sel) return UOCR_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(seq_lens, 4) || !aligned(sel, 4)) return UOCR_ERR_INVALID_ARG;
    if ((q_seq && !aligned(q_seq, 4)) || (q_pos && !aligned(q_pos, 4))) return UOCR_ERR_INVALID_ARG;
    if (dev_err && !aligned(dev_err, 4)) return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    uocr_status_t st;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_block_topk(c, scores, seq_lens, q_seq, q_pos, n_q, B, max_blocks,
                                               sel, dev_err));
}

uocr_status_t uocr_sparse_attn(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_table, const int32_t *seq_lens,
                               const int32_t *q_seq, const int32_t *q_pos, const int32_t *sel,
                               int n_q, int B, int H, int max_blocks, int num_pages, float scale,
                               void *out, int32_t *dev_err, uocr_stream_t stream) {
    uocr_status_t st = check_common(n_q, B, max_blocks, num_pages, block_table, seq_lens, q_seq,
                                    q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(out)) return UOCR_ERR_INVALID_ARG;
    if (!sel || !aligned(sel, 4)) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    if (!isfinite(scale)) return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_sparse_attn(c, q, k_cache, v_cache, block_table, seq_lens, q_seq,
                                                q_pos, sel, n_q, B, H, max_blocks, num_pages, scale,
                                                out, false, -1, false, dev_err));
}

}  // extern "C"

namespace uocr {
// Every check of uocr_sparse_decode that does not concern the workspace, in its order.
uocr_status_t check_sparse_decode_args(const void *q, const void *k_cache, const void *v_cache, const void *idx_q,
                                       const void *idx_k_cache, const int32_t *block_table,
                                       const int32_t *seq_lens, int B, int H, int max_blocks, int num_pages,
                                       const void *out, const int32_t *sel_out, const int32_t *dev_err) {
    uocr_status_t st = check_common(B, B, max_blocks, num_pages, block_table, seq_lens, nullptr,
                                    nullptr, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(out) || !bf16_ok(idx_q) ||
        !bf16_ok(idx_k_cache))
        return UOCR_ERR_INVALID_ARG;
    if (!sel_out || !aligned(sel_out, 4)) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    return UOCR_OK;
}
}  // namespace uocr

extern "C" {

uocr_status_t uocr_sparse_decode(const void *q, const void *k_cache, const void *v_cache,
                                 const void *idx_q, const void *idx_k_cache,
                                 const int32_t *block_table, const int32_t *seq_lens, int B, int H,
                                 int max_blocks, int num_pages, void *out, int32_t *sel_out,
                                 void *workspace, size_t workspace_bytes, int32_t *dev_err,
                                 uocr_stream_t stream) {
    uocr_status_t st = uocr::check_sparse_decode_args(q, k_cache, v_cache, idx_q, idx_k_cache, block_table,
                                                      seq_lens, B, H, max_blocks, num_pages, out, sel_out, dev_err);
    if (st != UOCR_OK) return st;
    const WsLayout w = ws_layout(B, H, max_blocks);
    if (!workspace || !aligned(workspace, kWsAlign) || workspace_bytes < w.total) return UOCR_ERR_WORKSPACE;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    char *ws = (char *)workspace;
    float *scores = (float *)(ws + w.scores_off);
    cudaError_t e = uocr::launch_index_scan(c, idx_q, idx_k_cache, block_table, seq_lens, nullptr,
                                            nullptr, B, B, max_blocks, num_pages, scores, dev_err);
    if (e != cudaSuccess) return cuda_status(e);
    c.pdl = true;
    e = uocr::launch_block_topk(c, scores, seq_lens, nullptr, nullptr, B, B, max_blocks, sel_out, dev_err);
    if (e != cudaSuccess) return cuda_status(e);
    const float scale = 1.0f / sqrtf((float)UOCR_HEAD_DIM);
    e = uocr::launch_sparse_attn(c, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, sel_out,
                                 B, B, H, max_blocks, num_pages, scale, out, true, -1, false, dev_err);
    return cuda_status(e);
}

uocr_status_t uocr_prefill_index_score(const void *idx_q, const void *idx_k_cache, const int32_t *block_table,
                                       const int32_t *seq_lens, int seq, const int32_t *q_pos, int n_q, int B,
                                       int max_blocks, int num_pages, float *scores, int32_t *dev_err,
                                       uocr_stream_t stream) {
    uocr_status_t st = check_common(n_q, B, max_blocks, num_pages, block_table, seq_lens, nullptr, q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(idx_q) || !bf16_ok(idx_k_cache) || !q_pos || !scores || !aligned(scores, 4))
        return UOCR_ERR_INVALID_ARG;
    if (seq < 0 || seq >= B) return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_prefill_index_gemm(c, idx_q, idx_k_cache, block_table + (size_t)seq * max_blocks,
                                                       seq_lens + seq, q_pos, n_q, max_blocks, num_pages, scores,
                                                       nullptr, dev_err));
}

size_t uocr_prefill_workspace_bytes(int n_q, int H, int max_blocks) {
    if (n_q <= 0 || H <= 0 || max_blocks <= 0) return 0;
    return ws_layout(n_q, H, max_blocks).total + uocr::prefill_attn_workspace(n_q, H, max_blocks, nullptr);
}

uocr_status_t uocr_sparse_prefill(const void *q, const void *k_cache, const void *v_cache, const void *idx_q,
                                  const void *idx_k_cache, const int32_t *block_table, const int32_t *seq_lens,
                                  int seq, const int32_t *q_pos, int n_q, int B, int H, int max_blocks,
                                  int num_pages, void *out, int32_t *sel_out, void *workspace,
                                  size_t workspace_bytes, int32_t *dev_err, uocr_stream_t stream) {
    uocr_status_t st = check_common(n_q, B, max_blocks, num_pages, block_table, seq_lens, nullptr, q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(out) || !bf16_ok(idx_q) ||
        !bf16_ok(idx_k_cache) || !q_pos)
        return UOCR_ERR_INVALID_ARG;
    if (!sel_out || !aligned(sel_out, 4)) return UOCR_ERR_INVALID_ARG;
    if (seq < 0 || seq >= B) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    if (n_q == 0) return UOCR_OK;
    if ((long long)n_q * UOCR_N_SEL > 0x7fffffffLL || (long long)n_q * H > 0x7fffffffLL) return UOCR_ERR_UNSUPPORTED;
    if ((long long)num_pages * H > 0x7fffffffLL) return UOCR_ERR_UNSUPPORTED;   // TMA tile coordinates are int32
    const WsLayout w = ws_layout(n_q, H, max_blocks);
    if (!workspace || !aligned(workspace, kWsAlign) || workspace_bytes < uocr_prefill_workspace_bytes(n_q, H, max_blocks))
        return UOCR_ERR_WORKSPACE;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    float *scores = (float *)((char *)workspace + w.scores_off);
    char *attn_ws = (char *)workspace + w.total;
    uocr::PrefillAttnWs aw;
    uocr::prefill_attn_workspace(n_q, H, max_blocks, &aw);
    cudaError_t e = cudaMemsetAsync(attn_ws, 0, aw.zero_bytes, c.stream);
    if (e != cudaSuccess) return cuda_status(e);
    const int32_t *bt_row = block_table + (size_t)seq * max_blocks;
    e = uocr::launch_prefill_index_gemm(c, idx_q, idx_k_cache, bt_row, seq_lens + seq, q_pos, n_q, max_blocks,
                                        num_pages, scores, (int32_t *)(attn_ws + aw.sched_off), dev_err);
    if (e != cudaSuccess) return cuda_status(e);
    c.pdl = true;
    e = uocr::launch_block_topk(c, scores, seq_lens, nullptr, q_pos, n_q, B, max_blocks, sel_out, dev_err, seq);
    if (e != cudaSuccess) return cuda_status(e);
    const float scale = 1.0f / sqrtf((float)UOCR_HEAD_DIM);
    e = uocr::launch_prefill_attn(c, q, k_cache, v_cache, bt_row, seq_lens + seq, q_pos, sel_out, n_q, H, max_blocks,
                                  num_pages, scale, out, attn_ws, dev_err);
    return cuda_status(e);
}

size_t uocr_sparse_attn_seq_workspace_bytes(int n_q, int H, int max_blocks) {
    if (n_q <= 0 || H <= 0 || max_blocks <= 0) return 0;
    return uocr::prefill_attn_workspace(n_q, H, max_blocks, nullptr);
}

uocr_status_t uocr_sparse_attn_seq(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_table, const int32_t *seq_lens, int seq,
                                   const int32_t *q_pos, const int32_t *sel, int n_q, int B, int H,
                                   int max_blocks, int num_pages, float scale, void *out, void *workspace,
                                   size_t workspace_bytes, int32_t *dev_err, uocr_stream_t stream) {
    uocr_status_t st = check_common(n_q, B, max_blocks, num_pages, block_table, seq_lens, nullptr, q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(out) || !q_pos) return UOCR_ERR_INVALID_ARG;
    if (!sel || !aligned(sel, 4)) return UOCR_ERR_INVALID_ARG;
    if (seq < 0 || seq >= B) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    if (!isfinite(scale)) return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    if ((long long)n_q * UOCR_N_SEL > 0x7fffffffLL || (long long)n_q * H > 0x7fffffffLL) return UOCR_ERR_UNSUPPORTED;
    if ((long long)num_pages * H > 0x7fffffffLL) return UOCR_ERR_UNSUPPORTED;   // TMA tile coordinates are int32
    if (!workspace || !aligned(workspace, kWsAlign) ||
        workspace_bytes < uocr_sparse_attn_seq_workspace_bytes(n_q, H, max_blocks))
        return UOCR_ERR_WORKSPACE;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    uocr::PrefillAttnWs aw;
    uocr::prefill_attn_workspace(n_q, H, max_blocks, &aw);
    char *ws = (char *)workspace;
    cudaError_t e = cudaMemsetAsync(ws, 0, aw.zero_bytes, c.stream);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(uocr::launch_prefill_attn(c, q, k_cache, v_cache, block_table + (size_t)seq * max_blocks,
                                                 seq_lens + seq, q_pos, sel, n_q, H, max_blocks, num_pages, scale, out,
                                                 workspace, dev_err));
}

size_t uocr_dense_workspace_bytes(int B, int H, int max_blocks) {
    if (B <= 0 || H <= 0 || max_blocks <= 0) return 0;
    return uocr::dense_attn_workspace(B, H, max_blocks);
}

uocr_status_t uocr_dense_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                                const int32_t *seq_lens, int ref_blocks, int B, int H, int max_blocks, int num_pages,
                                void *out, void *workspace, size_t workspace_bytes, int32_t *dev_err,
                                uocr_stream_t stream) {
    uocr_status_t st = check_common(B, B, max_blocks, num_pages, block_table, seq_lens, nullptr, nullptr, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(out)) return UOCR_ERR_INVALID_ARG;
    if (ref_blocks < 0) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    if (!workspace || !aligned(workspace, kWsAlign) || workspace_bytes < uocr_dense_workspace_bytes(B, H, max_blocks))
        return UOCR_ERR_WORKSPACE;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    const float scale = 1.0f / sqrtf((float)UOCR_HEAD_DIM);
    return cuda_status(uocr::launch_dense_attn(c, q, k_cache, v_cache, block_table, seq_lens, B, H, max_blocks,
                                               num_pages, ref_blocks, scale, out, workspace, dev_err));
}

uocr_status_t uocr_rope_append(void *q, void *idx_q, const void *k_new, const void *v_new, const void *idx_k_new,
                               const int32_t *tok_pos, const int32_t *page_pos, const int32_t *q_seq,
                               const int32_t *q_pos, const int32_t *block_table, const int32_t *seq_lens, int n,
                               int B, int H, int max_blocks, int num_pages, void *k_cache, void *v_cache,
                               void *idx_k_cache, int32_t *dev_err, uocr_stream_t stream) {
    uocr_status_t st = check_common(n, B, max_blocks, num_pages, block_table, seq_lens, q_seq, q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(idx_q) || !bf16_ok(k_new) || !bf16_ok(v_new) || !bf16_ok(idx_k_new) ||
        !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(idx_k_cache))
        return UOCR_ERR_INVALID_ARG;
    if (!tok_pos || !page_pos || !aligned(tok_pos, 4) || !aligned(page_pos, 4)) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    if (n == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_rope_append(c, q, idx_q, k_new, v_new, idx_k_new, tok_pos, page_pos, q_seq,
                                                q_pos, block_table, seq_lens, n, B, H, max_blocks, num_pages,
                                                k_cache, v_cache, idx_k_cache, dev_err));
}

uocr_status_t uocr_summary_score(const void *idx_q, const void *summary_cache, const int32_t *block_table,
                                 const int32_t *seq_lens, const int32_t *q_seq, const int32_t *q_pos, int n_q, int B,
                                 int max_blocks, int num_pages, float *scores, int32_t *dev_err,
                                 uocr_stream_t stream) {
    uocr_status_t st = check_common(n_q, B, max_blocks, num_pages, block_table, seq_lens, q_seq, q_pos, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(idx_q) || !bf16_ok(summary_cache) || !scores || !aligned(scores, 4)) return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_summary_scan(c, idx_q, summary_cache, block_table, seq_lens, q_seq, q_pos, n_q,
                                                 B, max_blocks, num_pages, scores, dev_err));
}

uocr_status_t uocr_block_summary_mean(const void *idx_k_cache, const int32_t *pages, int n_pages, int num_pages,
                                      void *summary_cache, int32_t *dev_err, uocr_stream_t stream) {
    if (!bf16_ok(idx_k_cache) || !bf16_ok(summary_cache) || n_pages < 0 || num_pages < 1) return UOCR_ERR_INVALID_ARG;
    if ((pages && !aligned(pages, 4)) || (dev_err && !aligned(dev_err, 4))) return UOCR_ERR_INVALID_ARG;
    if (n_pages == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    uocr_status_t st;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_block_mean(c, idx_k_cache, pages, n_pages, num_pages, summary_cache, dev_err));
}

uocr_status_t uocr_sparse_decode_summary(const void *q, const void *k_cache, const void *v_cache, const void *idx_q,
                                         const void *summary_cache, const int32_t *block_table,
                                         const int32_t *seq_lens, int B, int H, int max_blocks, int num_pages,
                                         void *out, int32_t *sel_out, void *workspace, size_t workspace_bytes,
                                         int32_t *dev_err, uocr_stream_t stream) {
    uocr_status_t st = check_common(B, B, max_blocks, num_pages, block_table, seq_lens, nullptr, nullptr, dev_err);
    if (st != UOCR_OK) return st;
    if (!bf16_ok(q) || !bf16_ok(k_cache) || !bf16_ok(v_cache) || !bf16_ok(out) || !bf16_ok(idx_q) ||
        !bf16_ok(summary_cache))
        return UOCR_ERR_INVALID_ARG;
    if (!sel_out || !aligned(sel_out, 4)) return UOCR_ERR_INVALID_ARG;
    if (H < 1 || H > UOCR_MAX_HEADS) return UOCR_ERR_UNSUPPORTED;
    const WsLayout w = ws_layout(B, H, max_blocks);
    if (!workspace || !aligned(workspace, kWsAlign) || workspace_bytes < w.total) return UOCR_ERR_WORKSPACE;
    uocr::LaunchCtx c;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    float *scores = (float *)((char *)workspace + w.scores_off);
    cudaError_t e = uocr::launch_summary_scan(c, idx_q, summary_cache, block_table, seq_lens, nullptr, nullptr, B, B,
                                              max_blocks, num_pages, scores, dev_err);
    if (e != cudaSuccess) return cuda_status(e);
    c.pdl = true;
    e = uocr::launch_block_topk(c, scores, seq_lens, nullptr, nullptr, B, B, max_blocks, sel_out, dev_err);
    if (e != cudaSuccess) return cuda_status(e);
    const float scale = 1.0f / sqrtf((float)UOCR_HEAD_DIM);
    e = uocr::launch_sparse_attn(c, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, sel_out, B, B, H,
                                 max_blocks, num_pages, scale, out, true, -1, false, dev_err);
    return cuda_status(e);
}

uocr_status_t uocr_block_topk_masked(const float *scores, const int32_t *seq_lens, const int32_t *q_seq,
                                     const int32_t *q_pos, const uint32_t *cand_mask, int mask_words, int n_q, int B,
                                     int max_blocks, int32_t *sel, int32_t *dev_err, uocr_stream_t stream) {
    if (n_q < 0 || B < 1 || max_blocks < 1) return UOCR_ERR_INVALID_ARG;
    if (!scores || !seq_lens || !sel || !cand_mask) return UOCR_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(seq_lens, 4) || !aligned(sel, 4) || !aligned(cand_mask, 4))
        return UOCR_ERR_INVALID_ARG;
    if ((q_seq && !aligned(q_seq, 4)) || (q_pos && !aligned(q_pos, 4))) return UOCR_ERR_INVALID_ARG;
    if (dev_err && !aligned(dev_err, 4)) return UOCR_ERR_INVALID_ARG;
    if ((long long)mask_words * 32 < (long long)max_blocks) return UOCR_ERR_INVALID_ARG;
    if (n_q == 0) return UOCR_OK;
    uocr::LaunchCtx c;
    uocr_status_t st;
    if ((st = make_ctx(stream, false, c)) != UOCR_OK) return st;
    return cuda_status(uocr::launch_block_topk(c, scores, seq_lens, q_seq, q_pos, n_q, B, max_blocks, sel, dev_err,
                                               -1, cand_mask, mask_words));
}

}  // extern "C"
