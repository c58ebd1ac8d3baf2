"""Parity of the chunked-prefill path (tcgen05 block scoring, selection, attention)
with the fp64 oracle, through the C ABI.

Small cases check every query and every block score; they span several
128-query and 256-token tiles with ragged tails (n_q not a multiple of 128,
contexts not a multiple of 256, shuffled pages).  The full chunked-prefill
workload (2048 queries over 65536 tokens) is checked on every query.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import OUT_MAX_ATOL, OUT_MEAN_ATOL, check_all_queries, check_queries, oracle_attend

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def uocr(cuda_device):
    import block_sparse_long_uocr_b200 as m
    return m


def _prefill_case(total, n_new, extra_pos=(), seed=0, shuffle=True, device="cpu", heads=10):
    pos = list(range(total - n_new, total)) + list(extra_pos)
    return workloads.make_case([total], q_seq=[0] * len(pos), q_pos=pos, shuffle=shuffle, seed=seed,
                               device=device, heads=heads)


@pytest.mark.parametrize("total,n_new,extra", [
    (300, 1, ()),                                  # one query, one partial N tile
    (1000, 5, (0, 31, 32, 255, 256, 257)),         # n_q < 128: shrunk A box
    (4096 + 17, 300, (0, 1, 4000)),                # 3 M tiles (ragged), 17 N tiles (ragged)
    (2048, 128, ()),                               # exactly one M tile
    (2048, 129, ()),                               # one query over
    (32768 + 5, 1100, ()),                         # 325 work units: 3 on some CTAs (the A ring wraps)
])
def test_prefill_scores_match_oracle(uocr, cuda_device, total, n_new, extra):
    case = _prefill_case(total, n_new, extra, seed=total + n_new, device=cuda_device, heads=1)
    sc = uocr.prefill_index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, 0, case.q_pos)
    torch.cuda.synchronize()
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos, want_out=False)
    got = sc.cpu().double().numpy()
    for i in range(case.n_q):
        nb = int(case.q_pos[i]) // 32 + 1
        np.testing.assert_allclose(got[i, :nb], r["scores"][i, :nb], rtol=0, atol=1e-3, err_msg=f"query {i}")
        assert np.isneginf(got[i, nb:]).all()          # not written past the causal blocks


def test_prefill_scores_agree_with_the_scan_kernel(uocr, cuda_device):
    case = _prefill_case(32 * 700 + 9, 260, seed=11, device=cuda_device, heads=1)
    a = uocr.prefill_index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, 0, case.q_pos)
    b = uocr.index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, case.q_seq, case.q_pos)
    torch.cuda.synchronize()
    fin = torch.isfinite(b)
    assert torch.equal(fin, torch.isfinite(a))
    assert (a[fin] - b[fin]).abs().max().item() <= 1e-3


def test_sparse_prefill_matches_oracle(uocr, cuda_device):
    """Tiles of consecutive positions (local windows on the tensor-core kernel) and a tile with
    scattered positions (its local entries on the block kernel); no device error on a clean call
    (a drain or pipeline wait that ran out would set UOCR_DEVERR_TIMEOUT)."""
    case = _prefill_case(4096, 300, (0, 31, 100, 511, 512, 513), seed=5, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, sel = uocr.sparse_prefill(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                                   case.seq_lens, 0, case.q_pos, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_queries(case, range(case.n_q), out, sel)


def test_sparse_prefill_second_sequence_and_paging(uocr, cuda_device):
    """Queries of sequence 1 of a 3-sequence batch with shuffled pages."""
    lens = [32 * 40, 32 * 90 + 3, 700]
    pos = list(range(lens[1] - 150, lens[1]))
    case = workloads.make_case(lens, q_seq=[1] * len(pos), q_pos=pos, shuffle=True, seed=9, device=cuda_device)
    out, sel = uocr.sparse_prefill(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                                   case.seq_lens, 1, case.q_pos)
    torch.cuda.synchronize()
    check_queries(case, range(case.n_q), out, sel)


def test_prefill_flags_bad_positions_and_pages(uocr, cuda_device):
    case = _prefill_case(2000, 40, seed=3, device=cuda_device, heads=1)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bad_pos = case.q_pos.clone()
    bad_pos[3] = 2000                                    # at the sequence length: invalid
    sc = uocr.prefill_index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, 0, bad_pos,
                                  dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_POS
    assert torch.isneginf(sc[3]).all()                   # nothing written for the invalid query
    err.zero_()
    bt = case.block_table.clone()
    bt[0, 7] = case.num_pages + 3
    sc = uocr.prefill_index_score(case.idx_q, case.idx_k_pool, bt, case.seq_lens, 0, case.q_pos, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_PAGE
    assert torch.isneginf(sc[:, 7]).all() and torch.isfinite(sc[:, 6]).all()


def test_prefill_scoring_wait_timeout_is_flagged_and_recovers(uocr, cuda_device):
    """The scoring GEMM's epilogue gives up its first accumulator wait at once: UOCR_DEVERR_TIMEOUT
    is set, every role of the CTA stops issuing, drains what it issued (the drain waits keep the
    default limit) and frees its TMEM, and the next call with the default limit matches the
    oracle."""
    import ctypes
    fn = uocr.lib.uocr_test_first_wait_limit_ns
    fn.argtypes = [ctypes.c_longlong]
    fn.restype = None
    case = _prefill_case(4096 + 17, 300, seed=23, device=cuda_device, heads=1)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    fn(0)
    try:
        uocr.prefill_index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, 0, case.q_pos,
                                 dev_err=err)
        torch.cuda.synchronize()
    finally:
        fn(-1)
    assert int(err.item()) & uocr.DEVERR_TIMEOUT
    err.zero_()
    sc = uocr.prefill_index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, 0, case.q_pos,
                                  dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos, want_out=False)
    got = sc.cpu().double().numpy()
    for i in range(case.n_q):
        nb = int(case.q_pos[i]) // 32 + 1
        np.testing.assert_allclose(got[i, :nb], r["scores"][i, :nb], rtol=0, atol=1e-3, err_msg=f"query {i}")


def test_sparse_prefill_bad_page_gives_an_empty_block(uocr, cuda_device):
    """A selected block whose page id is out of range is flagged and contributes nothing: every
    output equals exact attention over the query's other selected blocks."""
    total = 32 * 80
    case = _prefill_case(total, 100, seed=21, device=cuda_device)
    j_bad = (total - 1) // 32 - 2                       # in the local window of most queries
    bt = case.block_table.clone()
    bt[0, j_bad] = case.num_pages + 5
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, sel = uocr.sparse_prefill(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, bt,
                                   case.seq_lens, 0, case.q_pos, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_PAGE
    assert torch.isfinite(out.float()).all()
    got, sel = out.float().cpu().numpy(), sel.cpu().numpy()
    hit = 0
    for i in range(case.n_q):
        s = sel[i].copy()
        hit += int((s == j_bad).any())
        s[s == j_bad] = -1
        ref = oracle_attend(case, i, s)
        d = np.abs(got[i] - ref)
        assert d.max() <= OUT_MAX_ATOL and d.mean() <= OUT_MEAN_ATOL, f"query {i}"
    assert hit > 50


def _random_selection(case, seed, empty_frac=0.2):
    """Per query: distinct causal blocks (up to 16) in random slots, some slots empty (-1)."""
    g = np.random.default_rng(seed)
    sel = np.full((case.n_q, 16), -1, np.int32)
    for i in range(case.n_q):
        nb = int(case.q_pos[i]) // 32 + 1
        k = min(16, nb)
        picks = g.choice(nb, size=k, replace=False)
        keep = g.random(k) >= empty_frac
        keep[0] = True
        slots = g.permutation(16)[:k]
        sel[i, slots[keep]] = picks[keep]
    return sel


def test_sparse_attn_seq_matches_oracle(uocr, cuda_device):
    """Block-centric attention of a caller's selection (ragged n_q, several 16-entry items per
    block, empty slots, blocks shared by many queries) against the oracle, query by query."""
    case = _prefill_case(32 * 90 + 11, 333, (0, 5, 31, 32, 700), seed=31, device=cuda_device)
    sel = _random_selection(case, 31)
    sel_d = torch.from_numpy(sel).to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = uocr.sparse_attn_seq(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, 0, case.q_pos,
                               sel_d, dev_err=err)
    ref_q = uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, sel_d,
                             case.q_seq, case.q_pos)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.float().cpu().numpy()
    for i in range(case.n_q):
        ref = oracle_attend(case, i, sel[i])
        d = np.abs(got[i] - ref)
        assert d.max() <= OUT_MAX_ATOL and d.mean() <= OUT_MEAN_ATOL, f"query {i}"
    # and the query-centric entry on the same selection agrees to within both roundings
    assert (out.float() - ref_q.float()).abs().max().item() <= 2e-2


def test_sparse_attn_seq_reuses_one_workspace(uocr, cuda_device):
    """Consecutive calls on one workspace, each checked against the oracle on its own selection.
    The merge drops the partials it has read from L2, leaving their memory undefined; a call
    writes every slot it uses before its merge reads it, so a slot that was empty in one call and
    selected in the next (and the reverse) must not carry anything over."""
    case = _prefill_case(32 * 70 + 7, 200, (0, 31, 64), seed=41, device=cuda_device)
    mb = int(case.block_table.shape[1])
    ws = torch.empty(uocr.sparse_attn_seq_workspace_bytes(case.n_q, 10, mb), dtype=torch.uint8,
                     device=cuda_device)
    first = _random_selection(case, 41, empty_frac=0.5)
    second = _random_selection(case, 42, empty_frac=0.0)
    third = second.copy()
    third[:, 1::2] = -1                                 # slots full in the second call, empty now
    none = (third < 0).all(axis=1)
    third[none] = second[none]                          # a query keeps at least one block
    for sel in (first, second, third, first):
        out = uocr.sparse_attn_seq(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, 0,
                                   case.q_pos, torch.from_numpy(sel).to(cuda_device), workspace=ws)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        for i in range(case.n_q):
            ref = oracle_attend(case, i, sel[i])
            d = np.abs(got[i] - ref)
            assert d.max() <= OUT_MAX_ATOL and d.mean() <= OUT_MEAN_ATOL, f"query {i}"


@pytest.mark.parametrize("heads", [1, 3])
def test_sparse_attn_seq_odd_head_counts(uocr, cuda_device, heads):
    """Head counts for which a head-parity split of the block kernel's work would hand consecutive
    uses of a ring stage to different producers: every output against the oracle, no device error
    (a pipeline wait that passed on an older phase would show as wrong outputs or a timeout)."""
    case = _prefill_case(32 * 300, 1200, seed=51 + heads, device=cuda_device, heads=heads)
    sel = _random_selection(case, 51 + heads, empty_frac=0.0)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = uocr.sparse_attn_seq(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, 0, case.q_pos,
                               torch.from_numpy(sel).to(cuda_device), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.float().cpu().numpy()
    for i in range(case.n_q):
        d = np.abs(got[i] - oracle_attend(case, i, sel[i]))
        assert d.max() <= OUT_MAX_ATOL and d.mean() <= OUT_MEAN_ATOL, f"query {i}"


def test_sparse_attn_seq_flags_bad_selections(uocr, cuda_device):
    case = _prefill_case(32 * 40, 64, seed=32, device=cuda_device, heads=3)
    sel = _random_selection(case, 32, empty_frac=0.0)
    sel[5, 3] = int(case.q_pos[5]) // 32 + 1           # one block past the query's causal range
    q_pos = case.q_pos.clone()
    q_pos[7] = int(case.seq_lens[0])                    # a position at the sequence length: invalid
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = uocr.sparse_attn_seq(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, 0, q_pos,
                               torch.from_numpy(sel).to(cuda_device), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_SEL and int(err.item()) & uocr.DEVERR_POS
    assert not int(err.item()) & uocr.DEVERR_TIMEOUT
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all() and (got[7] == 0).all()
    s5 = sel[5].copy()
    s5[3] = -1
    for i, s in ((5, s5), (6, sel[6])):
        d = np.abs(got[i] - oracle_attend(case, i, s))
        assert d.max() <= OUT_MAX_ATOL and d.mean() <= OUT_MEAN_ATOL, f"query {i}"


@pytest.mark.slow
def test_chunked_prefill_workload_every_query(uocr, cuda_device):
    """The chunked-prefill workload as the bench runs it (2048 queries over 65536 tokens): every
    tensor-core block score, every selection and every output against the oracle."""
    case = workloads.chunked_prefill(device=cuda_device)
    ws = uocr.alloc_prefill_workspace(case.n_q, 10, case.max_blocks, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, sel = uocr.sparse_prefill(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                                   case.seq_lens, 0, case.q_pos, workspace=ws, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    scores = ws[: case.n_q * case.max_blocks * 4].view(torch.float32).view(case.n_q, case.max_blocks)
    check_all_queries(case, out, sel, scores)


@pytest.mark.slow
def test_long_chunk_twelve_heads_every_query(uocr, cuda_device):
    """A 4096-query chunk starting 7 tokens into a block, 12 heads, shuffled pages: 32 local-window
    tiles of 8-block windows x 12 heads = 384 units for the local kernel's CTAs (about 11 each), the
    block kernel's units from its counter beside them, and 49152 (query, head) merges; every
    selection and every output against the oracle, no device error."""
    total = 32 * 400 + 7
    case = _prefill_case(total, 4096, seed=61, device=cuda_device, heads=12)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, sel = uocr.sparse_prefill(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                                   case.seq_lens, 0, case.q_pos, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_all_queries(case, out, sel)
