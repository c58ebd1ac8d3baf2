"""TEST INFRASTRUCTURE: the fp64 CPU oracle of the SR-SWA / DASH block-sparse step.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline``
leg may import this package.  The product (``block_sparse_long_uocr_b200``)
never imports it, and it never imports the product: the two share nothing but
the seeded input generators in ``workloads``.

The arithmetic lives in ``uocr_oracle.c`` (plain C, fp64, OpenMP over queries);
this module only compiles it with gcc and marshals numpy arrays.  Each wrapper
cites the page section its C function follows:

* [rkmt 五 steps 1-2] block score = max over the block's tokens of q_idx . k_idx
  (Unlimited-OCR-2 walk-through, news.rkmt.cn/news/25027, section 五);
* [rkmt 五 step 3], [lqnn 显存账本] 4 local blocks + top-12 remote blocks
  (www.lqnn.cn/news/271890, section 显存账本);
* [rkmt 五 step 4], [chenxutan 2.3.2] exact softmax attention over the selected
  tokens (chenxutan.com/d/4261.html, section 2.3.2, scaled dot product);
* [rkmt 四], [rkmt 六] page2d rotary embedding (63 frequency pairs on the in-page
  token offset, theta 10000, resampled over the full spectrum; 1 pair on the
  page coordinate page % 2, theta 256) applied before the new token's keys are
  appended to the paged caches;
* [lqnn 显存账本], [leheaven 二] block-summary scoring (one summary vector per block)
  and the mean-key summary; [rkmt 五] selection under a page-aware candidate mask.

Parity status: pinned (tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "uocr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Method constants as the pages give them ([rkmt 五], [rkmt 三], [lqnn 显存账本]).
BLOCK = 32          # sparse_block_size
N_LOCAL = 4         # sparse_local_block (4 x 32 = 128-token local window)
N_REMOTE = 12       # dash_topk_blocks
N_SEL = N_LOCAL + N_REMOTE   # sparse_topk_blocks = 16
HEADS = 10          # num_attention_heads = num_key_value_heads (MHA)
HEAD_DIM = 128
IDX_DIM = 128       # one indexer head of 128 dims
TIE_EPS = 1e-3      # near-tie band on the 12th/13th remote score gap
# page2d rotary embedding ([rkmt 四], [rkmt 六]): 1 of the 64 frequency pairs on the page axis
ROPE_PAGE_PAIRS = 1     # sparse_rope_page_pairs
ROPE_THETA_TOK = 10000.0
ROPE_THETA_PAGE = 256.0
ROPE_PAGE_MOD = 2       # sparse_rope_page_mod: page coordinate = page % 2


def build(force: bool = False) -> str:
    """Compile uocr_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
            return _LIB
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fopenmp", "-fPIC",
               "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
        return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dd = ctypes.c_double
        lib.uocr_oracle_num_causal_blocks.argtypes = [I, I]
        lib.uocr_oracle_num_causal_blocks.restype = I
        lib.uocr_oracle_block_scores.argtypes = [P, P, P, I, I, I, P]
        lib.uocr_oracle_block_scores.restype = I
        lib.uocr_oracle_select.argtypes = [P, I, I, I, Dd, P, P]
        lib.uocr_oracle_select.restype = I
        lib.uocr_oracle_attend.argtypes = [P, P, P, P, P, I, I, I, I, I, Dd, P]
        lib.uocr_oracle_attend.restype = None
        lib.uocr_oracle_run.argtypes = ([I, P, P, P, P, P, P, P, P] + [I] * 7
                                        + [Dd, Dd, P, P, P, P, P, I])
        lib.uocr_oracle_run.restype = I
        L = ctypes.c_longlong
        lib.uocr_oracle_rope_page2d.argtypes = [P, I, I, Dd, Dd, I, L, L, P]
        lib.uocr_oracle_rope_page2d.restype = None
        lib.uocr_oracle_summary_scores.argtypes = [P, P, P, I, I, I, P]
        lib.uocr_oracle_summary_scores.restype = I
        lib.uocr_oracle_block_mean.argtypes = [P, I, I, I, P]
        lib.uocr_oracle_block_mean.restype = None
        lib.uocr_oracle_select_masked.argtypes = [P, I, I, I, P, Dd, P, P]
        lib.uocr_oracle_select_masked.restype = I
        _lib = lib
    return _lib


# --------------------------------------------------------------------------- marshalling
def bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of the bit patterns."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy input must hold bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected a bf16 tensor, got {x.dtype}")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def ints(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.int32)
    return np.ascontiguousarray(x.detach().cpu().numpy().astype(np.int32))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def decode_positions(seq_lens, q_seq) -> np.ndarray:
    """Decode reading: the query of sequence b is its last cached token, p = seq_len_b - 1."""
    sl = ints(seq_lens)
    return (sl[ints(q_seq)] - 1).astype(np.int32)


# --------------------------------------------------------------------------- per-step wrappers
def num_causal_blocks(p: int, blk: int = BLOCK) -> int:
    return int(_load().uocr_oracle_num_causal_blocks(int(p), int(blk)))


def block_scores(idx_q_row, idx_k_pool, bt_row, p: int, blk: int = BLOCK) -> np.ndarray:
    """[rkmt 五 steps 1-2] fp64 scores of the causal blocks of one query (length nb)."""
    qi = bits(idx_q_row).reshape(-1)
    kp = bits(idx_k_pool)
    bt = ints(bt_row).reshape(-1)
    d_idx = qi.shape[0]
    assert kp.shape[-1] == d_idx and kp.shape[-2] == blk
    nb = num_causal_blocks(p, blk)
    s = np.empty(max(nb, 1), dtype=np.float64)
    _load().uocr_oracle_block_scores(_ptr(qi), _ptr(kp), _ptr(bt), int(p), int(blk), int(d_idx), _ptr(s))
    return s[:nb]


def select(scores, nb: int, n_local: int = N_LOCAL, n_remote: int = N_REMOTE,
           tie_eps: float = TIE_EPS):
    """[rkmt 五 step 3] -> (sel ascending, -1 padded, to n_local+n_remote; near_tie flag)."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64).reshape(-1))
    assert s.shape[0] >= nb
    sel = np.empty(n_local + n_remote, dtype=np.int32)
    tie = ctypes.c_int(0)
    _load().uocr_oracle_select(_ptr(s if s.size else np.zeros(1)), int(nb), int(n_local), int(n_remote),
                               float(tie_eps), _ptr(sel), ctypes.byref(tie))
    return sel, bool(tie.value)


def attend(q_row, k_pool, v_pool, bt_row, sel, p: int, blk: int = BLOCK, scale: float | None = None):
    """[rkmt 五 step 4] fp64 softmax attention of one query ([H, D]) over the selected blocks."""
    qb = bits(q_row)
    H, D = qb.shape
    kp, vp = bits(k_pool), bits(v_pool)
    assert kp.shape[1:] == (H, blk, D) and vp.shape == kp.shape
    s = ints(sel).reshape(-1)
    bt = ints(bt_row).reshape(-1)
    sc = float(scale) if scale is not None else 1.0 / np.sqrt(D)
    out = np.empty((H, D), dtype=np.float64)
    _load().uocr_oracle_attend(_ptr(qb), _ptr(kp), _ptr(vp), _ptr(bt), _ptr(s), int(s.shape[0]), int(p),
                               int(H), int(D), int(blk), sc, _ptr(out))
    return out


# --------------------------------------------------------------------------- whole step
def run(q, idx_q, k_pool, v_pool, idx_k_pool, block_table, q_seq, q_pos, *,
        blk: int = BLOCK, n_local: int = N_LOCAL, n_remote: int = N_REMOTE,
        scale: float | None = None, tie_eps: float = TIE_EPS, sel_in=None,
        want_scores: bool = True, want_out: bool = True, threads: int = 0) -> dict:
    """The whole step for n_q queries (OpenMP over queries).

    q [n_q,H,D], idx_q [n_q,d_idx] bf16; k_pool / v_pool [P,H,blk,D],
    idx_k_pool [P,blk,d_idx] bf16; block_table [B,max_blocks] int32;
    q_seq, q_pos [n_q] int32.  Returns a dict with ``scores`` [n_q,max_blocks]
    fp64 (-inf past the causal blocks), ``sel`` [n_q,n_local+n_remote] int32,
    ``near_tie`` [n_q] bool, ``out`` [n_q,H,D] fp64 and ``threads``.
    With ``sel_in`` the selection is taken as given (scores / near_tie are then None).
    """
    qb, qib = bits(q), bits(idx_q)
    kp, vp, ikp = bits(k_pool), bits(v_pool), bits(idx_k_pool)
    bt = ints(block_table)
    qs, qp = ints(q_seq).reshape(-1), ints(q_pos).reshape(-1)
    n_q = qs.shape[0]
    H, D = qb.shape[1], qb.shape[2]
    d_idx = qib.shape[1]
    max_blocks = bt.shape[1]
    n_sel = n_local + n_remote
    sc = float(scale) if scale is not None else 1.0 / np.sqrt(D)
    scores = np.empty((n_q, max_blocks), np.float64) if (want_scores and sel_in is None) else None
    tie = np.zeros(n_q, np.int32) if sel_in is None else None
    sel = np.empty((n_q, n_sel), np.int32)
    out = np.empty((n_q, H, D), np.float64) if want_out else None
    si = ints(sel_in) if sel_in is not None else None
    used = _load().uocr_oracle_run(
        int(n_q), _ptr(qs), _ptr(qp), _ptr(qb), _ptr(qib), _ptr(kp), _ptr(vp), _ptr(ikp), _ptr(bt),
        int(max_blocks), int(H), int(D), int(d_idx), int(blk), int(n_local), int(n_remote),
        sc, float(tie_eps), _ptr(si), _ptr(scores), _ptr(sel), _ptr(tie), _ptr(out), int(threads))
    return {"scores": scores, "sel": sel, "near_tie": None if tie is None else tie.astype(bool),
            "out": out, "threads": int(used)}


# --------------------------------------------------------------------------- page2d rotary + cache append
def rope_page2d(x, tok: int, page: int, *, page_pairs: int = ROPE_PAGE_PAIRS, theta_tok: float = ROPE_THETA_TOK,
                theta_page: float = ROPE_THETA_PAGE, page_mod: int = ROPE_PAGE_MOD) -> np.ndarray:
    """[rkmt 四] fp64 page2d rotation of one bf16 vector (last dim = 2 * pairs) -> float64 array."""
    xb = bits(x).reshape(-1)
    n_pairs = xb.shape[0] // 2
    out = np.empty(2 * n_pairs, dtype=np.float64)
    _load().uocr_oracle_rope_page2d(_ptr(xb), int(n_pairs), int(page_pairs), float(theta_tok), float(theta_page),
                                    int(page_mod), int(tok), int(page), _ptr(out))
    return out


def rope_append(q, idx_q, k_new, v_new, idx_k_new, tok_pos, page_pos, seqs, positions, block_table,
                k_cache, v_cache, idx_k_cache):
    """The step before the scan, for n new tokens: rotate q, idx_q, k_new, idx_k_new with page2d and
    write k, v, idx_k of token i into the caches at (sequence seqs[i], position positions[i]).
    Returns (q_rot, idx_q_rot, k_cache, v_cache, idx_k_cache) as float64 arrays (caches copied)."""
    qb, qib = bits(q), bits(idx_q)
    kb, vb, ikb = bits(k_new), bits(v_new), bits(idx_k_new)
    tp, pp = ints(tok_pos).reshape(-1), ints(page_pos).reshape(-1)
    sq, ps = ints(seqs).reshape(-1), ints(positions).reshape(-1)
    bt = ints(block_table)
    kc = bits(k_cache).astype(np.uint32)
    n, H = qb.shape[0], qb.shape[1]
    blk = kc.shape[2]

    def widen(a):
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    kcache, vcache, icache = widen(bits(k_cache)), widen(bits(v_cache)), widen(bits(idx_k_cache))
    q_rot = np.empty(qb.shape, np.float64)
    qi_rot = np.empty(qib.shape, np.float64)
    for i in range(n):
        t, g = int(tp[i]), int(pp[i])
        for h in range(H):
            q_rot[i, h] = rope_page2d(qb[i, h], t, g)
        qi_rot[i] = rope_page2d(qib[i], t, g)
        page = int(bt[sq[i], ps[i] // blk])
        row = int(ps[i]) % blk
        for h in range(H):
            kcache[page, h, row] = rope_page2d(kb[i, h], t, g)
            vcache[page, h, row] = widen(vb[i, h])
        icache[page, row] = rope_page2d(ikb[i], t, g)
    del kc
    return q_rot, qi_rot, kcache, vcache, icache


# --------------------------------------------------------------------------- summary scoring, masked selection
def summary_scores(idx_q_row, summary_pool, bt_row, p: int, blk: int = BLOCK) -> np.ndarray:
    """fp64 scores of the causal blocks from one summary vector per page ([P, d_idx] bf16)."""
    qi = bits(idx_q_row).reshape(-1)
    sp = bits(summary_pool)
    bt = ints(bt_row).reshape(-1)
    nb = num_causal_blocks(p, blk)
    s = np.empty(max(nb, 1), dtype=np.float64)
    _load().uocr_oracle_summary_scores(_ptr(qi), _ptr(sp), _ptr(bt), int(p), int(blk), int(qi.shape[0]), _ptr(s))
    return s[:nb]


def block_mean(idx_k_pool, page: int) -> np.ndarray:
    kp = bits(idx_k_pool)
    blk, d_idx = kp.shape[1], kp.shape[2]
    out = np.empty(d_idx, dtype=np.float64)
    _load().uocr_oracle_block_mean(_ptr(kp), int(page), int(blk), int(d_idx), _ptr(out))
    return out


def select_masked(scores, nb: int, mask_words, n_local: int = N_LOCAL, n_remote: int = N_REMOTE,
                  tie_eps: float = TIE_EPS):
    """Selection where only remote candidates with their mask bit set may be picked."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64).reshape(-1))
    m = np.ascontiguousarray(np.asarray(mask_words, dtype=np.uint32).reshape(-1))
    sel = np.empty(n_local + n_remote, dtype=np.int32)
    tie = ctypes.c_int(0)
    _load().uocr_oracle_select_masked(_ptr(s if s.size else np.zeros(1)), int(nb), int(n_local), int(n_remote),
                                      _ptr(m if m.size else np.zeros(1, np.uint32)), float(tie_eps), _ptr(sel),
                                      ctypes.byref(tie))
    return sel, bool(tie.value)
