// decode_static.cu -- uocr_sparse_decode_static: the decode step with no
// caller-provided workspace and no allocation of any kind.
//
// Some callers cannot allocate device memory at the point where they decode:
// a plugin running inside a host engine that owns every device allocation, or
// a latency-critical decode loop where a cudaMalloc (which may synchronise the
// device) is not allowed.  For them this entry point keeps its scratch (the
// fp32 block scores [B][max_blocks]; the attention merges its split-K partials
// on chip and needs none) in one file-scope device array of
// UOCR_STATIC_SCRATCH_BYTES, which every GPU that loads the library holds until
// the process exits.
//
// The array's host-side name is only a stand-in for the symbol, not a device
// address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it; later calls
// reuse it.  Nothing in the scratch has to start at zero: every score the
// kernels read is written earlier in the same call.  The argument checks run
// in the order of uocr_sparse_decode's and the scratch size is tested after
// them, so a call returns the status uocr_sparse_decode would.  All calls on a
// device share the one array, so calls whose kernels overlap on the GPU
// (different streams, or concurrent host threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "uocr.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[UOCR_STATIC_SCRATCH_BYTES];

std::once_flag g_once[kMaxDevices];
void *g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_status[kMaxDevices];

}  // namespace

extern "C" uocr_status_t uocr_sparse_decode_static(
    const void *q, const void *k_cache, const void *v_cache, const void *idx_q, const void *idx_k_cache,
    const int32_t *block_table, const int32_t *seq_lens, int B, int H, int max_blocks, int num_pages,
    void *out, int32_t *sel_out, int32_t *dev_err, uocr_stream_t stream) {
    const uocr_status_t st = uocr::check_sparse_decode_args(q, k_cache, v_cache, idx_q, idx_k_cache, block_table,
                                                            seq_lens, B, H, max_blocks, num_pages, out, sel_out,
                                                            dev_err);
    if (st != UOCR_OK) return st;
    if (uocr_workspace_bytes(B, H, max_blocks) > (size_t)UOCR_STATIC_SCRATCH_BYTES)
        return UOCR_ERR_WORKSPACE;   // needs more scratch than the static array holds

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return UOCR_ERR_CUDA;
    std::call_once(g_once[dev], [dev] {
        g_scratch_status[dev] = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_static_scratch);
    });
    if (g_scratch_status[dev] != cudaSuccess || g_scratch_ptr[dev] == nullptr) return UOCR_ERR_CUDA;

    return uocr_sparse_decode(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, B, H, max_blocks,
                              num_pages, out, sel_out, g_scratch_ptr[dev], (size_t)UOCR_STATIC_SCRATCH_BYTES,
                              dev_err, stream);
}
