"""Python binding of libuocr.so, the B200 (sm_100a) SR-SWA / DASH block-sparse attention step.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/uocr.h``.  PyTorch provides the
device memory and the stream; there is no CPU fallback: the first call (or
any access to ``lib``) raises ``ImportError`` when ``libuocr.so`` has not been
built (``python -m block_sparse_long_uocr_b200.build``).  The library is loaded
on first use so that the build module can be imported before it exists.

Entry points (same names as the C ABI, without the ``uocr_`` prefix):

* :func:`index_score`  -- block scores of the 1-head x 128 Lightning Indexer;
* :func:`block_topk`   -- 4 local + top-12 remote block selection;
* :func:`sparse_attn`  -- exact 10-head attention over the selected 512 tokens;
* :func:`sparse_decode` -- the three fused into one decode call;
* :func:`prefill_index_score` -- the block scores of a prefill chunk on the tcgen05 tensor cores;
* :func:`sparse_prefill` -- tensor-core scoring, selection and attention for a prefill chunk;
* :func:`sparse_attn_seq` -- the block-centric attention of many queries of one sequence over a
  caller's selection (the attention stage of :func:`sparse_prefill`);
* :func:`summary_score`, :func:`block_summary_mean`, :func:`sparse_decode_summary` -- block-summary
  scoring (one vector per block) and the decode step built on it;
* :func:`block_topk_masked` -- selection under a page-aware candidate bitmap;
* :func:`rope_append` -- page2d rotary embedding of new tokens and their append to the caches;
* :func:`dense_decode` -- comparator: full causal attention, or an R-SWA-style reference
  prefix plus the 128-token window (the baselines the sparse step is measured against);
* :func:`sparse_decode_static` -- the same decode call for callers that cannot
  allocate device memory (scratch held inside the library);
* :func:`workspace_bytes`.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libuocr.so")

BLOCK = 32
N_LOCAL = 4
N_REMOTE = 12
N_SEL = 16
HEAD_DIM = 128
IDX_DIM = 128

STATUS = {0: "UOCR_OK", 1: "UOCR_ERR_INVALID_ARG", 2: "UOCR_ERR_UNSUPPORTED",
          3: "UOCR_ERR_WORKSPACE", 4: "UOCR_ERR_CUDA"}
DEVERR_PAGE, DEVERR_POS, DEVERR_SEL, DEVERR_TIMEOUT = 1, 2, 4, 8


class UocrError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_uocr_b200.build` "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.uocr_status_string.argtypes = [I]
    lib.uocr_status_string.restype = ctypes.c_char_p
    lib.uocr_abi_version.argtypes = []
    lib.uocr_abi_version.restype = I
    lib.uocr_last_cuda_error.argtypes = []
    lib.uocr_last_cuda_error.restype = ctypes.c_char_p
    lib.uocr_workspace_bytes.argtypes = [I, I, I]
    lib.uocr_workspace_bytes.restype = Z
    lib.uocr_index_score.argtypes = [P, P, P, P, P, P, I, I, I, I, P, P, P]
    lib.uocr_index_score.restype = I
    lib.uocr_block_topk.argtypes = [P, P, P, P, I, I, I, P, P, P]
    lib.uocr_block_topk.restype = I
    lib.uocr_sparse_attn.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, P]
    lib.uocr_sparse_attn.restype = I
    lib.uocr_sparse_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, P, P, Z, P, P]
    lib.uocr_sparse_decode.restype = I
    lib.uocr_summary_score.argtypes = [P, P, P, P, P, P, I, I, I, I, P, P, P]
    lib.uocr_summary_score.restype = I
    lib.uocr_block_summary_mean.argtypes = [P, P, I, I, P, P, P]
    lib.uocr_block_summary_mean.restype = I
    lib.uocr_sparse_decode_summary.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, P, P, Z, P, P]
    lib.uocr_sparse_decode_summary.restype = I
    lib.uocr_block_topk_masked.argtypes = [P, P, P, P, P, I, I, I, I, P, P, P]
    lib.uocr_block_topk_masked.restype = I
    lib.uocr_rope_append.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, P, P]
    lib.uocr_rope_append.restype = I
    lib.uocr_dense_workspace_bytes.argtypes = [I, I, I]
    lib.uocr_dense_workspace_bytes.restype = Z
    lib.uocr_dense_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, P, P]
    lib.uocr_dense_decode.restype = I
    lib.uocr_prefill_workspace_bytes.argtypes = [I, I, I]
    lib.uocr_prefill_workspace_bytes.restype = Z
    lib.uocr_prefill_index_score.argtypes = [P, P, P, P, I, P, I, I, I, I, P, P, P]
    lib.uocr_prefill_index_score.restype = I
    lib.uocr_sparse_prefill.argtypes = [P, P, P, P, P, P, P, I, P, I, I, I, I, I, P, P, P, Z, P, P]
    lib.uocr_sparse_prefill.restype = I
    lib.uocr_sparse_attn_seq_workspace_bytes.argtypes = [I, I, I]
    lib.uocr_sparse_attn_seq_workspace_bytes.restype = Z
    lib.uocr_sparse_attn_seq.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, F, P, P, Z, P, P]
    lib.uocr_sparse_attn_seq.restype = I
    lib.uocr_sparse_decode_static.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, P, P, P]
    lib.uocr_sparse_decode_static.restype = I
    return lib


_LIB = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _lib()
    raise AttributeError(name)


# --------------------------------------------------------------------------- helpers
def _check(fn: str, st: int):
    if st != 0:
        msg = _lib().uocr_status_string(st).decode()
        if st == 4:   # UOCR_ERR_CUDA: name the CUDA error behind it
            msg += f" ({_lib().uocr_last_cuda_error().decode()})"
        raise UocrError(fn, st, msg)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int | None = None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _opt_i32(t, name, n=None):
    if t is None:
        return None
    _dev(t, name, torch.int32, 1)
    if n is not None:
        _shape(t, name, (n,))
    return t


def _shape(t: torch.Tensor, name: str, shape) -> torch.Tensor:
    """Refuse, before any launch, a tensor whose shape differs from what the kernels will index
    (None in `shape` accepts any extent): a smaller buffer would be written or read past its end
    on the device."""
    got = tuple(t.shape)
    if len(got) != len(shape) or any(e is not None and g != e for g, e in zip(got, shape)):
        want = "[" + ", ".join("*" if e is None else str(e) for e in shape) + "]"
        raise ValueError(f"{name} must have shape {want}, got {list(got)}")
    return t


def _check_caches(k_cache, v_cache, H):
    """K / V caches [P, H, 32, 128] of the same shape."""
    _shape(k_cache, "k_cache", (None, H, BLOCK, HEAD_DIM))
    _shape(v_cache, "v_cache", tuple(k_cache.shape))


def _check_decode_args(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, out, sel):
    """One decode query per sequence: every per-sequence tensor has B rows, the caches agree on
    the head count and the pool size, and the outputs match the queries."""
    B, H = q.shape[0], q.shape[1]
    _shape(q, "q", (B, H, HEAD_DIM))
    _check_caches(k_cache, v_cache, H)
    _shape(idx_q, "idx_q", (B, IDX_DIM))
    if idx_k_cache is not None:
        _shape(idx_k_cache, "idx_k_cache", (k_cache.shape[0], BLOCK, IDX_DIM))
    _shape(block_table, "block_table", (B, None))
    _shape(seq_lens, "seq_lens", (B,))
    if out is not None:
        _shape(out, "out", (B, H, HEAD_DIM))
    if sel is not None:
        _shape(sel, "sel", (B, N_SEL))


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_bytes(n_q: int, heads: int, max_blocks: int) -> int:
    return int(_lib().uocr_workspace_bytes(int(n_q), int(heads), int(max_blocks)))


def prefill_workspace_bytes(n_q: int, heads: int, max_blocks: int) -> int:
    return int(_lib().uocr_prefill_workspace_bytes(int(n_q), int(heads), int(max_blocks)))


def alloc_prefill_workspace(n_q: int, heads: int, max_blocks: int, device) -> torch.Tensor:
    """uint8 workspace for sparse_prefill; its first n_q*max_blocks*4 bytes hold the block scores."""
    return torch.empty(max(prefill_workspace_bytes(n_q, heads, max_blocks), 1), dtype=torch.uint8, device=device)


def sparse_attn_seq_workspace_bytes(n_q: int, heads: int, max_blocks: int) -> int:
    return int(_lib().uocr_sparse_attn_seq_workspace_bytes(int(n_q), int(heads), int(max_blocks)))


def alloc_workspace(n_q: int, heads: int, max_blocks: int, device) -> torch.Tensor:
    """A uint8 tensor of workspace_bytes(...) bytes (torch allocations are 256-byte aligned)."""
    return torch.empty(max(workspace_bytes(n_q, heads, max_blocks), 1), dtype=torch.uint8, device=device)


# --------------------------------------------------------------------------- entry points
def index_score(idx_q, idx_k_cache, block_table, seq_lens, q_seq=None, q_pos=None, *,
                scores=None, dev_err=None, stream=None) -> torch.Tensor:
    """fp32 [n_q, max_blocks] block scores (entries past a query's causal blocks untouched)."""
    _dev(idx_q, "idx_q", torch.bfloat16, 2)
    _dev(idx_k_cache, "idx_k_cache", torch.bfloat16, 3)
    _dev(block_table, "block_table", torch.int32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    n_q, B, mb = idx_q.shape[0], block_table.shape[0], block_table.shape[1]
    _shape(idx_q, "idx_q", (n_q, IDX_DIM))
    _shape(idx_k_cache, "idx_k_cache", (None, BLOCK, IDX_DIM))
    _shape(seq_lens, "seq_lens", (B,))
    if scores is None:
        scores = torch.full((n_q, mb), float("-inf"), dtype=torch.float32, device=idx_q.device)
    _dev(scores, "scores", torch.float32, 2)
    _shape(scores, "scores", (n_q, mb))
    _check("uocr_index_score", _lib().uocr_index_score(
        _ptr(idx_q), _ptr(idx_k_cache), _ptr(block_table), _ptr(seq_lens), _ptr(_opt_i32(q_seq, "q_seq", n_q)),
        _ptr(_opt_i32(q_pos, "q_pos", n_q)), n_q, B, mb, idx_k_cache.shape[0], _ptr(scores),
        _ptr(dev_err), _stream(stream)))
    return scores


def block_topk(scores, seq_lens, q_seq=None, q_pos=None, *, sel=None, dev_err=None, stream=None) -> torch.Tensor:
    """int32 [n_q, 16] selected logical blocks (ascending, -1 padded)."""
    _dev(scores, "scores", torch.float32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    n_q, mb = scores.shape
    if sel is None:
        sel = torch.empty((n_q, N_SEL), dtype=torch.int32, device=scores.device)
    _dev(sel, "sel", torch.int32, 2)
    _shape(sel, "sel", (n_q, N_SEL))
    _check("uocr_block_topk", _lib().uocr_block_topk(
        _ptr(scores), _ptr(seq_lens), _ptr(_opt_i32(q_seq, "q_seq", n_q)), _ptr(_opt_i32(q_pos, "q_pos", n_q)),
        n_q, seq_lens.shape[0], mb, _ptr(sel), _ptr(dev_err), _stream(stream)))
    return sel


def sparse_attn(q, k_cache, v_cache, block_table, seq_lens, sel, q_seq=None, q_pos=None, *,
                scale: float | None = None, out=None, dev_err=None, stream=None) -> torch.Tensor:
    """bf16 [n_q, H, 128] attention output over the selected blocks."""
    _dev(q, "q", torch.bfloat16, 3)
    _dev(k_cache, "k_cache", torch.bfloat16, 4)
    _dev(v_cache, "v_cache", torch.bfloat16, 4)
    _dev(block_table, "block_table", torch.int32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    _dev(sel, "sel", torch.int32, 2)
    n_q, H = q.shape[0], q.shape[1]
    B, mb = block_table.shape
    _shape(q, "q", (n_q, H, HEAD_DIM))
    _check_caches(k_cache, v_cache, H)
    _shape(seq_lens, "seq_lens", (B,))
    _shape(sel, "sel", (n_q, N_SEL))
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, 3)
    _shape(out, "out", (n_q, H, HEAD_DIM))
    sc = float(scale) if scale is not None else HEAD_DIM ** -0.5
    _check("uocr_sparse_attn", _lib().uocr_sparse_attn(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
        _ptr(_opt_i32(q_seq, "q_seq", n_q)), _ptr(_opt_i32(q_pos, "q_pos", n_q)), _ptr(sel), n_q, B, H, mb,
        k_cache.shape[0], ctypes.c_float(sc), _ptr(out), _ptr(dev_err), _stream(stream)))
    return out


def sparse_decode(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, *,
                  out=None, sel=None, workspace=None, dev_err=None, stream=None):
    """One decode query per sequence at p = seq_len - 1.  Returns (out [B,H,128] bf16, sel [B,16] int32)."""
    _dev(q, "q", torch.bfloat16, 3)
    _dev(k_cache, "k_cache", torch.bfloat16, 4)
    _dev(v_cache, "v_cache", torch.bfloat16, 4)
    _dev(idx_q, "idx_q", torch.bfloat16, 2)
    _dev(idx_k_cache, "idx_k_cache", torch.bfloat16, 3)
    _dev(block_table, "block_table", torch.int32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, H = q.shape[0], q.shape[1]
    mb = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if sel is None:
        sel = torch.empty((B, N_SEL), dtype=torch.int32, device=q.device)
    _dev(out, "out", torch.bfloat16, 3)
    _dev(sel, "sel", torch.int32, 2)
    _check_decode_args(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, out, sel)
    if workspace is None:
        workspace = alloc_workspace(B, H, mb, q.device)
    _check("uocr_sparse_decode", _lib().uocr_sparse_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx_q), _ptr(idx_k_cache), _ptr(block_table),
        _ptr(seq_lens), B, H, mb, k_cache.shape[0], _ptr(out), _ptr(sel), _ptr(workspace),
        workspace.numel(), _ptr(dev_err), _stream(stream)))
    return out, sel


def prefill_index_score(idx_q, idx_k_cache, block_table, seq_lens, seq: int, q_pos, *,
                        scores=None, dev_err=None, stream=None) -> torch.Tensor:
    """fp32 [n_q, max_blocks] block scores of n_q queries of sequence `seq` (tcgen05 GEMM)."""
    _dev(idx_q, "idx_q", torch.bfloat16, 2)
    _dev(idx_k_cache, "idx_k_cache", torch.bfloat16, 3)
    _dev(block_table, "block_table", torch.int32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    _dev(q_pos, "q_pos", torch.int32, 1)
    n_q, B, mb = idx_q.shape[0], block_table.shape[0], block_table.shape[1]
    _shape(idx_q, "idx_q", (n_q, IDX_DIM))
    _shape(idx_k_cache, "idx_k_cache", (None, BLOCK, IDX_DIM))
    _shape(seq_lens, "seq_lens", (B,))
    _shape(q_pos, "q_pos", (n_q,))
    if scores is None:
        scores = torch.full((n_q, mb), float("-inf"), dtype=torch.float32, device=idx_q.device)
    _dev(scores, "scores", torch.float32, 2)
    _shape(scores, "scores", (n_q, mb))
    _check("uocr_prefill_index_score", _lib().uocr_prefill_index_score(
        _ptr(idx_q), _ptr(idx_k_cache), _ptr(block_table), _ptr(seq_lens), int(seq), _ptr(q_pos), n_q, B, mb,
        idx_k_cache.shape[0], _ptr(scores), _ptr(dev_err), _stream(stream)))
    return scores


def sparse_prefill(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, seq: int, q_pos, *,
                   out=None, sel=None, workspace=None, dev_err=None, stream=None):
    """Prefill chunk of sequence `seq`.  Returns (out [n_q,H,128] bf16, sel [n_q,16] int32)."""
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 3), (k_cache, "k_cache", torch.bfloat16, 4),
                         (v_cache, "v_cache", torch.bfloat16, 4), (idx_q, "idx_q", torch.bfloat16, 2),
                         (idx_k_cache, "idx_k_cache", torch.bfloat16, 3), (block_table, "block_table", torch.int32, 2),
                         (seq_lens, "seq_lens", torch.int32, 1), (q_pos, "q_pos", torch.int32, 1)):
        _dev(t, n, dt, nd)
    n_q, H = q.shape[0], q.shape[1]
    B, mb = block_table.shape
    if out is None:
        out = torch.empty_like(q)
    if sel is None:
        sel = torch.empty((n_q, N_SEL), dtype=torch.int32, device=q.device)
    _dev(out, "out", torch.bfloat16, 3)
    _dev(sel, "sel", torch.int32, 2)
    _shape(q, "q", (n_q, H, HEAD_DIM))
    _check_caches(k_cache, v_cache, H)
    _shape(idx_q, "idx_q", (n_q, IDX_DIM))
    _shape(idx_k_cache, "idx_k_cache", (k_cache.shape[0], BLOCK, IDX_DIM))
    _shape(seq_lens, "seq_lens", (B,))
    _shape(q_pos, "q_pos", (n_q,))
    _shape(out, "out", (n_q, H, HEAD_DIM))
    _shape(sel, "sel", (n_q, N_SEL))
    if workspace is None:
        workspace = alloc_prefill_workspace(n_q, H, mb, q.device)
    _check("uocr_sparse_prefill", _lib().uocr_sparse_prefill(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx_q), _ptr(idx_k_cache), _ptr(block_table), _ptr(seq_lens),
        int(seq), _ptr(q_pos), n_q, B, H, mb, k_cache.shape[0], _ptr(out), _ptr(sel), _ptr(workspace),
        workspace.numel(), _ptr(dev_err), _stream(stream)))
    return out, sel


def sparse_attn_seq(q, k_cache, v_cache, block_table, seq_lens, seq: int, q_pos, sel, *, scale=None,
                    out=None, workspace=None, dev_err=None, stream=None) -> torch.Tensor:
    """Attention of many queries of sequence `seq` over the given selection (block-centric).
    Returns out [n_q,H,128] bf16."""
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 3), (k_cache, "k_cache", torch.bfloat16, 4),
                         (v_cache, "v_cache", torch.bfloat16, 4), (block_table, "block_table", torch.int32, 2),
                         (seq_lens, "seq_lens", torch.int32, 1), (q_pos, "q_pos", torch.int32, 1),
                         (sel, "sel", torch.int32, 2)):
        _dev(t, n, dt, nd)
    n_q, H = q.shape[0], q.shape[1]
    B, mb = block_table.shape
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, 3)
    _shape(q, "q", (n_q, H, HEAD_DIM))
    _check_caches(k_cache, v_cache, H)
    _shape(seq_lens, "seq_lens", (B,))
    _shape(q_pos, "q_pos", (n_q,))
    _shape(sel, "sel", (n_q, N_SEL))
    _shape(out, "out", (n_q, H, HEAD_DIM))
    if workspace is None:
        workspace = torch.empty(max(sparse_attn_seq_workspace_bytes(n_q, H, mb), 1), dtype=torch.uint8,
                                device=q.device)
    sc = float(scale) if scale is not None else HEAD_DIM ** -0.5
    _check("uocr_sparse_attn_seq", _lib().uocr_sparse_attn_seq(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), int(seq), _ptr(q_pos), _ptr(sel),
        n_q, B, H, mb, k_cache.shape[0], sc, _ptr(out), _ptr(workspace), workspace.numel(), _ptr(dev_err),
        _stream(stream)))
    return out


def summary_score(idx_q, summary_cache, block_table, seq_lens, q_seq=None, q_pos=None, *,
                  scores=None, dev_err=None, stream=None) -> torch.Tensor:
    """fp32 [n_q, max_blocks]: idx_q . summary of each causal block's page."""
    _dev(idx_q, "idx_q", torch.bfloat16, 2)
    _dev(summary_cache, "summary_cache", torch.bfloat16, 2)
    _dev(block_table, "block_table", torch.int32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    n_q, B, mb = idx_q.shape[0], block_table.shape[0], block_table.shape[1]
    _shape(idx_q, "idx_q", (n_q, IDX_DIM))
    _shape(summary_cache, "summary_cache", (None, IDX_DIM))
    _shape(seq_lens, "seq_lens", (B,))
    if scores is None:
        scores = torch.full((n_q, mb), float("-inf"), dtype=torch.float32, device=idx_q.device)
    _dev(scores, "scores", torch.float32, 2)
    _shape(scores, "scores", (n_q, mb))
    _check("uocr_summary_score", _lib().uocr_summary_score(
        _ptr(idx_q), _ptr(summary_cache), _ptr(block_table), _ptr(seq_lens), _ptr(_opt_i32(q_seq, "q_seq", n_q)),
        _ptr(_opt_i32(q_pos, "q_pos", n_q)), n_q, B, mb, summary_cache.shape[0], _ptr(scores), _ptr(dev_err),
        _stream(stream)))
    return scores


def block_summary_mean(idx_k_cache, summary_cache=None, pages=None, *, dev_err=None, stream=None) -> torch.Tensor:
    """bf16 [P, 128]: the mean of each (listed) page's indexer keys."""
    _dev(idx_k_cache, "idx_k_cache", torch.bfloat16, 3)
    P = idx_k_cache.shape[0]
    _shape(idx_k_cache, "idx_k_cache", (P, BLOCK, IDX_DIM))
    if summary_cache is None:
        summary_cache = torch.zeros((P, IDX_DIM), dtype=torch.bfloat16, device=idx_k_cache.device)
    _dev(summary_cache, "summary_cache", torch.bfloat16, 2)
    _shape(summary_cache, "summary_cache", (P, IDX_DIM))
    n = P if pages is None else _dev(pages, "pages", torch.int32, 1).shape[0]
    _check("uocr_block_summary_mean", _lib().uocr_block_summary_mean(
        _ptr(idx_k_cache), _ptr(pages), n, P, _ptr(summary_cache), _ptr(dev_err), _stream(stream)))
    return summary_cache


def sparse_decode_summary(q, k_cache, v_cache, idx_q, summary_cache, block_table, seq_lens, *,
                          out=None, sel=None, workspace=None, dev_err=None, stream=None):
    """sparse_decode with block-summary scoring.  Returns (out, sel)."""
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 3), (k_cache, "k_cache", torch.bfloat16, 4),
                         (v_cache, "v_cache", torch.bfloat16, 4), (idx_q, "idx_q", torch.bfloat16, 2),
                         (summary_cache, "summary_cache", torch.bfloat16, 2), (block_table, "block_table", torch.int32, 2),
                         (seq_lens, "seq_lens", torch.int32, 1)):
        _dev(t, n, dt, nd)
    B, H = q.shape[0], q.shape[1]
    mb = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if sel is None:
        sel = torch.empty((B, N_SEL), dtype=torch.int32, device=q.device)
    _dev(out, "out", torch.bfloat16, 3)
    _dev(sel, "sel", torch.int32, 2)
    _shape(summary_cache, "summary_cache", (k_cache.shape[0], IDX_DIM))
    _check_decode_args(q, k_cache, v_cache, idx_q, None, block_table, seq_lens, out, sel)
    if workspace is None:
        workspace = alloc_workspace(B, H, mb, q.device)
    _check("uocr_sparse_decode_summary", _lib().uocr_sparse_decode_summary(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx_q), _ptr(summary_cache), _ptr(block_table), _ptr(seq_lens),
        B, H, mb, k_cache.shape[0], _ptr(out), _ptr(sel), _ptr(workspace), workspace.numel(), _ptr(dev_err),
        _stream(stream)))
    return out, sel


def block_topk_masked(scores, seq_lens, cand_mask, q_seq=None, q_pos=None, *, sel=None, dev_err=None,
                      stream=None) -> torch.Tensor:
    """Selection where remote candidate j of sequence b needs bit j of cand_mask[b] (int32 words)."""
    _dev(scores, "scores", torch.float32, 2)
    _dev(seq_lens, "seq_lens", torch.int32, 1)
    _dev(cand_mask, "cand_mask", torch.int32, 2)
    n_q, mb = scores.shape
    _shape(cand_mask, "cand_mask", (seq_lens.shape[0], None))
    if sel is None:
        sel = torch.empty((n_q, N_SEL), dtype=torch.int32, device=scores.device)
    _dev(sel, "sel", torch.int32, 2)
    _shape(sel, "sel", (n_q, N_SEL))
    _check("uocr_block_topk_masked", _lib().uocr_block_topk_masked(
        _ptr(scores), _ptr(seq_lens), _ptr(_opt_i32(q_seq, "q_seq", n_q)), _ptr(_opt_i32(q_pos, "q_pos", n_q)),
        _ptr(cand_mask), cand_mask.shape[1], n_q, seq_lens.shape[0], mb, _ptr(sel), _ptr(dev_err), _stream(stream)))
    return sel


def rope_append(q, idx_q, k_new, v_new, idx_k_new, tok_pos, page_pos, block_table, seq_lens,
                k_cache, v_cache, idx_k_cache, q_seq=None, q_pos=None, *, dev_err=None, stream=None):
    """Rotate q / idx_q in place (page2d) and write the new tokens' rotated k / idx_k and raw v into the
    caches at each token's position (default: its sequence's last cached position)."""
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 3), (idx_q, "idx_q", torch.bfloat16, 2),
                         (k_new, "k_new", torch.bfloat16, 3), (v_new, "v_new", torch.bfloat16, 3),
                         (idx_k_new, "idx_k_new", torch.bfloat16, 2), (tok_pos, "tok_pos", torch.int32, 1),
                         (page_pos, "page_pos", torch.int32, 1), (block_table, "block_table", torch.int32, 2),
                         (seq_lens, "seq_lens", torch.int32, 1), (k_cache, "k_cache", torch.bfloat16, 4),
                         (v_cache, "v_cache", torch.bfloat16, 4), (idx_k_cache, "idx_k_cache", torch.bfloat16, 3)):
        _dev(t, n, dt, nd)
    n, H = q.shape[0], q.shape[1]
    B, mb = block_table.shape
    _shape(q, "q", (n, H, HEAD_DIM))
    _shape(idx_q, "idx_q", (n, IDX_DIM))
    _shape(k_new, "k_new", (n, H, HEAD_DIM))
    _shape(v_new, "v_new", (n, H, HEAD_DIM))
    _shape(idx_k_new, "idx_k_new", (n, IDX_DIM))
    _shape(tok_pos, "tok_pos", (n,))
    _shape(page_pos, "page_pos", (n,))
    _shape(seq_lens, "seq_lens", (B,))
    _check_caches(k_cache, v_cache, H)
    _shape(idx_k_cache, "idx_k_cache", (k_cache.shape[0], BLOCK, IDX_DIM))
    _check("uocr_rope_append", _lib().uocr_rope_append(
        _ptr(q), _ptr(idx_q), _ptr(k_new), _ptr(v_new), _ptr(idx_k_new), _ptr(tok_pos), _ptr(page_pos),
        _ptr(_opt_i32(q_seq, "q_seq", n)), _ptr(_opt_i32(q_pos, "q_pos", n)), _ptr(block_table), _ptr(seq_lens),
        n, B, H, mb, k_cache.shape[0], _ptr(k_cache), _ptr(v_cache), _ptr(idx_k_cache), _ptr(dev_err),
        _stream(stream)))
    return q, idx_q


def dense_workspace_bytes(n_q: int, heads: int, max_blocks: int) -> int:
    return int(_lib().uocr_dense_workspace_bytes(int(n_q), int(heads), int(max_blocks)))


def dense_decode(q, k_cache, v_cache, block_table, seq_lens, *, ref_blocks: int | None = None,
                 out=None, workspace=None, dev_err=None, stream=None) -> torch.Tensor:
    """Decode attention over blocks [0, ref_blocks) plus the 4-block local window (all blocks when
    ref_blocks is None: full causal attention).  Returns out [B,H,128] bf16."""
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 3), (k_cache, "k_cache", torch.bfloat16, 4),
                         (v_cache, "v_cache", torch.bfloat16, 4), (block_table, "block_table", torch.int32, 2),
                         (seq_lens, "seq_lens", torch.int32, 1)):
        _dev(t, n, dt, nd)
    B, H = q.shape[0], q.shape[1]
    mb = block_table.shape[1]
    rb = mb if ref_blocks is None else int(ref_blocks)
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.bfloat16, 3)
    _shape(q, "q", (B, H, HEAD_DIM))
    _check_caches(k_cache, v_cache, H)
    _shape(block_table, "block_table", (B, None))
    _shape(seq_lens, "seq_lens", (B,))
    _shape(out, "out", (B, H, HEAD_DIM))
    if workspace is None:
        workspace = torch.empty(max(dense_workspace_bytes(B, H, mb), 1), dtype=torch.uint8, device=q.device)
    _check("uocr_dense_decode", _lib().uocr_dense_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), rb, B, H, mb, k_cache.shape[0],
        _ptr(out), _ptr(workspace), workspace.numel(), _ptr(dev_err), _stream(stream)))
    return out


STATIC_SCRATCH_BYTES = 8 << 20   # UOCR_STATIC_SCRATCH_BYTES


def sparse_decode_static(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, *,
                         out, sel, dev_err=None, stream=None):
    """Decode without a workspace, for callers that cannot allocate device memory.

    The caller passes the outputs (`out` [B,H,128] bf16, `sel` [B,16] int32); the scratch
    lives in one fixed-size device array inside libuocr.so, shared by every call on the
    device (calls that overlap on the GPU race on it), so nothing is allocated here or in
    the library.  Raises UocrError (UOCR_ERR_WORKSPACE) when the shapes need more scratch
    than STATIC_SCRATCH_BYTES.  The first call on a device looks the array up; make it
    before any stream capture.
    """
    for t, n, dt, nd in ((q, "q", torch.bfloat16, 3), (k_cache, "k_cache", torch.bfloat16, 4),
                         (v_cache, "v_cache", torch.bfloat16, 4), (idx_q, "idx_q", torch.bfloat16, 2),
                         (idx_k_cache, "idx_k_cache", torch.bfloat16, 3), (block_table, "block_table", torch.int32, 2),
                         (seq_lens, "seq_lens", torch.int32, 1), (out, "out", torch.bfloat16, 3),
                         (sel, "sel", torch.int32, 2)):
        _dev(t, n, dt, nd)
    _check_decode_args(q, k_cache, v_cache, idx_q, idx_k_cache, block_table, seq_lens, out, sel)
    B, H = q.shape[0], q.shape[1]
    _check("uocr_sparse_decode_static", _lib().uocr_sparse_decode_static(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx_q), _ptr(idx_k_cache), _ptr(block_table),
        _ptr(seq_lens), B, H, block_table.shape[1], k_cache.shape[0], _ptr(out), _ptr(sel),
        _ptr(dev_err), _stream(stream)))
    return out, sel
