"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Every case, the full-size workloads included, is checked on every query and
every block score (the long-decode workload on every query of its first, a
middle and its last layer; the oracle reads back only each query's pages).
Tolerances: scores 1e-3 absolute; outputs 2e-2 max and
2e-3 mean absolute error; selections exact except oracle-flagged near ties.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import check_all_queries, check_queries

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def uocr(cuda_device):
    import block_sparse_long_uocr_b200 as m
    return m


def run_decode(uocr, case, layer=0, scores=True):
    """The decode call on one layer of a valid case; a clean call sets no device error bit."""
    q, qi = case.q_layers[layer]
    kp, vp, ikp = case.layers[layer]
    err = torch.zeros(1, dtype=torch.int32, device=q.device)
    sc = uocr.index_score(qi, ikp, case.block_table, case.seq_lens) if scores else None
    out, sel = uocr.sparse_decode(q, kp, vp, qi, ikp, case.block_table, case.seq_lens, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out, sel, sc


# ----------------------------------------------------------------------------- step by step
def test_index_score_matches_oracle_on_ragged_tails(uocr, cuda_device):
    lens = [1, 31, 32, 33, 100, 129, 500, 1000, 2047, 4100, 32 * 300 + 17]
    case = workloads.make_case(lens, shuffle=True, seed=3, device=cuda_device)
    sc = uocr.index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens)
    torch.cuda.synchronize()
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos, want_out=False)
    for b, L in enumerate(lens):
        nb = (L - 1) // 32 + 1
        np.testing.assert_allclose(sc[b, :nb].cpu().double().numpy(), r["scores"][b, :nb], rtol=0, atol=1e-3)
        # entries past the causal blocks are left as they were (-inf from the binding's fill)
        assert torch.isneginf(sc[b, nb:]).all()


@pytest.mark.parametrize("mb", [4096, 4093, 1021])
@pytest.mark.parametrize("kind", ["ties", "normal", "neg", "binary"])
def test_block_topk_is_exact_on_given_scores(uocr, cuda_device, kind, mb):
    """Few rows: one CTA per row.  Rows of up to 8 x 512 candidates are held in registers (odd
    row lengths start off a 16-byte boundary: scalar reads); 'normal' leaves a few dozen
    survivors (ranked by one warp), 'ties' hundreds (ranked by the CTA), 'binary' more than the
    survivor list holds (exact fallback)."""
    g = torch.Generator().manual_seed({"ties": 1, "normal": 2, "neg": 3, "binary": 4}[kind] + mb)
    lens = [1, 128, 129, 512, 513, 544, 545, 1000, 32 * 1024, 32 * 4096, 77777]
    if kind == "ties":
        s = torch.randint(-4, 5, (len(lens), mb), generator=g).float()
    elif kind == "normal":
        s = torch.randn(len(lens), mb, generator=g)
    elif kind == "binary":
        s = (torch.rand(len(lens), mb, generator=g) < 0.6).float()
    else:
        s = -torch.rand(len(lens), mb, generator=g) - 1.0
    lens = [min(L, mb * 32) for L in lens]
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    sel = uocr.block_topk(s.to(cuda_device), seq_lens.to(cuda_device))
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        nb = (L - 1) // 32 + 1
        want, _ = oracle.select(s[b].double().numpy(), nb)
        assert sel[b].cpu().tolist() == want.tolist(), f"row {b} (nb={nb})"


@pytest.mark.parametrize("kind,mb", [("ties", 1024), ("normal", 1023), ("neg", 1024), ("ties", 1021)])
def test_block_topk_many_rows_is_exact(uocr, cuda_device, kind, mb):
    """Enough rows for the warp-per-row selection; odd row lengths give rows that start off a
    16-byte boundary (scalar reads), 'ties' overflows the survivor list (exact fallback)."""
    g = torch.Generator().manual_seed({"ties": 11, "normal": 12, "neg": 13}[kind] + mb)
    n = 600
    edge = [1, 128, 129, 512, 513, 544, 545, 1000, 32 * mb]
    lens = edge + torch.randint(1, 32 * mb + 1, (n - len(edge),), generator=g).tolist()
    if kind == "ties":
        s = torch.randint(-4, 5, (n, mb), generator=g).float()
    elif kind == "normal":
        s = torch.randn(n, mb, generator=g)
    else:
        s = -torch.rand(n, mb, generator=g) - 1.0
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    sel = uocr.block_topk(s.to(cuda_device), seq_lens.to(cuda_device)).cpu()
    for b, L in enumerate(lens):
        nb = (L - 1) // 32 + 1
        want, _ = oracle.select(s[b].double().numpy(), nb)
        assert sel[b].tolist() == want.tolist(), f"row {b} (nb={nb})"


@pytest.mark.parametrize("heads", [1, 3, 10])
def test_sparse_attn_matches_oracle(uocr, cuda_device, heads):
    lens = [1, 40, 128, 129, 600, 32 * 64, 32 * 100 + 5]
    case = workloads.make_case(lens, heads=heads, shuffle=True, seed=5, device=cuda_device)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    sel = torch.from_numpy(r["sel"]).to(cuda_device)
    out = uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, sel)
    torch.cuda.synchronize()
    d = np.abs(out.float().cpu().numpy() - r["out"])
    assert d.max() <= 2e-2 and d.mean() <= 2e-3, (d.max(), d.mean())


def test_sparse_attn_custom_scale_and_partial_selection(uocr, cuda_device):
    case = workloads.make_case([32 * 40 + 3], heads=10, seed=6, device=cuda_device)
    sel_np = np.array([[1, 5, 9, 20, 36, 37, 38, 39, 40, -1, -1, -1, -1, -1, -1, -1]], np.int32)
    for scale in (0.0, 0.05, 0.3):
        out = uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens,
                               torch.from_numpy(sel_np).to(cuda_device), scale=scale)
        r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                       case.q_seq, case.q_pos, sel_in=sel_np, scale=scale)
        d = np.abs(out.float().cpu().numpy() - r["out"])
        assert d.max() <= 2e-2 and d.mean() <= 2e-3


def test_prefill_positions_through_the_step_entry_points(uocr, cuda_device):
    """Queries at arbitrary positions of one sequence (q_seq / q_pos given)."""
    pos = list(range(4096 - 300, 4096)) + [0, 31, 32, 127, 128, 511, 512, 513]
    case = workloads.make_case([4096], q_seq=[0] * len(pos), q_pos=pos, seed=7, device=cuda_device)
    sc = uocr.index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, case.q_seq, case.q_pos)
    sel = uocr.block_topk(sc, case.seq_lens, case.q_seq, case.q_pos)
    out = uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, sel,
                           case.q_seq, case.q_pos)
    torch.cuda.synchronize()
    check_queries(case, range(case.n_q), out, sel, sc)


# ----------------------------------------------------------------------------- fused decode
def test_decode_tiny_workload(uocr, cuda_device):
    case = workloads.tiny_decode(device=cuda_device)
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, range(case.n_q), out, sel, sc)


def test_decode_batched_planted_workload(uocr, cuda_device):
    case = workloads.batched_decode(device=cuda_device)
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, range(case.n_q), out, sel, sc)
    for b in range(16):
        assert sel[b, :12].cpu().tolist() == sorted(case.planted[b])
        assert sel[b, 12:].cpu().tolist() == list(range(1020, 1024))


@pytest.mark.parametrize("lens", [
    [1, 2, 31, 32, 33, 64, 127, 128, 129, 130],
    [511, 512, 513, 544, 545, 546, 576, 577, 1023, 1025],
])
def test_decode_edge_lengths(uocr, cuda_device, lens):
    case = workloads.make_case(lens, shuffle=True, seed=len(lens) + lens[0], device=cuda_device)
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, range(case.n_q), out, sel, sc)


def test_decode_small_ragged_shuffled(uocr, cuda_device):
    lens = workloads.ragged_lengths(9, 1, 300, seed=4)
    lens = [L - k for L, k in zip(lens, [0, 1, 5, 17, 31, 0, 2, 30, 9])]
    case = workloads.make_case(lens, shuffle=True, max_blocks=320, seed=4, device=cuda_device)
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, range(case.n_q), out, sel, sc)


def test_decode_empty_sequence_gives_zeros(uocr, cuda_device):
    case = workloads.make_case([64, 64], seed=1, device=cuda_device)
    seq_lens = torch.tensor([0, 64], dtype=torch.int32, device=cuda_device)
    out, sel = uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool,
                                  case.block_table, seq_lens)
    torch.cuda.synchronize()
    assert (sel[0] == -1).all() and (out[0] == 0).all()
    assert sel[1].tolist() == [0, 1] + [-1] * 14


def test_decode_is_deterministic(uocr, cuda_device):
    case = workloads.make_case([32 * 700, 32 * 900 + 5], shuffle=True, seed=8, device=cuda_device)
    o1, s1, _ = run_decode(uocr, case, scores=False)
    o2, s2, _ = run_decode(uocr, case, scores=False)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_decode_in_a_cuda_graph(uocr, cuda_device):
    case = workloads.make_case([32 * 300, 32 * 257 + 3, 5000], shuffle=True, seed=9, device=cuda_device)
    ws = uocr.alloc_workspace(3, 10, case.max_blocks, cuda_device)
    out = torch.empty_like(case.q)
    sel = torch.empty((3, 16), dtype=torch.int32, device=cuda_device)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                           case.seq_lens, out=out, sel=sel, workspace=ws)
    torch.cuda.synchronize()
    ref_out, ref_sel = out.clone(), sel.clone()
    out.zero_()
    sel.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
                           case.seq_lens, out=out, sel=sel, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(sel, ref_sel)


def test_device_errors_are_flagged_not_trapped(uocr, cuda_device):
    case = workloads.make_case([32 * 40, 32 * 40], seed=10, device=cuda_device)
    bt = case.block_table.clone()
    bt[0, 5] = case.num_pages + 7           # out of the pool: the kernels skip it and flag it
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, sel = uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, bt,
                                  case.seq_lens, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_PAGE
    assert 5 not in sel[0].tolist()          # its score is -inf: never selected while others remain
    # the untouched sequence is still right
    check_queries(case, [1], out, sel)

    err.zero_()
    long_lens = torch.tensor([32 * 40, 32 * 41], dtype=torch.int32, device=cuda_device)   # > 32 * max_blocks
    out, sel = uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool,
                                  case.block_table, long_lens, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_POS
    assert (sel[1] == -1).all() and (out[1] == 0).all()
    assert torch.isfinite(out.float()).all()


def _first_wait_limit(uocr, ns):
    """Test hook of the library (not in uocr.h): the limit of the first bounded wait of the decode
    attention and of the scoring GEMM's epilogue; 0 gives up at once, -1 restores the default."""
    import ctypes
    fn = uocr.lib.uocr_test_first_wait_limit_ns
    fn.argtypes = [ctypes.c_longlong]
    fn.restype = None
    fn(int(ns))


def test_decode_attention_wait_timeout_is_flagged_and_recovers(uocr, cuda_device):
    """The decode attention's wait for its V copy gives up at once: every block is dropped and
    UOCR_DEVERR_TIMEOUT is set, the kernel still drains its copies and ends, the outputs are finite
    (zeros: no block contributes), and the next call with the default limit matches the oracle."""
    case = workloads.make_case([32 * 300 + 5, 32 * 40, 700], shuffle=True, seed=12, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _first_wait_limit(uocr, 0)
    try:
        out, sel = uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool,
                                      case.block_table, case.seq_lens, dev_err=err)
        torch.cuda.synchronize()
    finally:
        _first_wait_limit(uocr, -1)
    assert int(err.item()) & uocr.DEVERR_TIMEOUT
    assert torch.isfinite(out.float()).all() and (out == 0).all()
    err.zero_()
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, range(case.n_q), out, sel, sc)


def test_binding_refuses_wrong_output_shapes_before_launching(uocr, cuda_device):
    """A selection buffer of 12 slots or an output of the wrong shape is refused by the binding
    with nothing launched (the caller's buffers keep their contents)."""
    case = workloads.make_case([32 * 64, 32 * 70], seed=13, device=cuda_device)
    B = case.n_q
    bad_sel = torch.full((B, 12), -5, dtype=torch.int32, device=cuda_device)
    out = torch.full_like(case.q, 3.0)
    sel = torch.full((B, 16), -5, dtype=torch.int32, device=cuda_device)
    bad_out = torch.full((B, 10, 64), 3.0, dtype=torch.bfloat16, device=cuda_device)
    for fn in (uocr.sparse_decode, uocr.sparse_decode_static):
        with pytest.raises(ValueError, match="sel"):
            fn(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens,
               out=out, sel=bad_sel)
        with pytest.raises(ValueError, match="out"):
            fn(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens,
               out=bad_out, sel=sel)
        with pytest.raises(ValueError, match="seq_lens"):
            fn(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool, case.block_table,
               case.seq_lens[:1].contiguous(), out=out, sel=sel)
    with pytest.raises(ValueError, match="sel"):
        uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, bad_sel)
    torch.cuda.synchronize()
    assert (bad_sel == -5).all() and (sel == -5).all() and (out == 3.0).all() and (bad_out == 3.0).all()


# ----------------------------------------------------------------------------- full-size workloads
@pytest.mark.slow
def test_decode_long_context_workload_every_query(uocr, cuda_device):
    """The long-decode workload as the bench runs it (16 sequences x 131072 tokens, 12 layer caches,
    126 GiB): every query of the first, a middle and the last layer against the oracle."""
    case = workloads.long_decode(device=cuda_device)
    for layer in (0, 5, 11):
        out, sel, sc = run_decode(uocr, case, layer=layer)
        check_queries(case, range(case.n_q), out, sel, sc, layer=layer)
    del case
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_decode_ragged_paged_workload_every_query(uocr, cuda_device):
    case = workloads.ragged_paged_decode(device=cuda_device)
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, range(case.n_q), out, sel, sc)
    del case
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_decode_maximum_lengths(uocr, cuda_device):
    """A 1.6M-token row (50,000 blocks: past the selection's shared-memory staging of 49,152
    candidates, so it reads its scores from L2), a 1M-token row (32,768 blocks, staged), and a
    short row sharing the same block table width."""
    lens = [32 * 50000, 32 * 32768 - 5, 700]
    case = workloads.make_case(lens, shuffle=True, max_blocks=50000, seed=17, device=cuda_device)
    out, sel, sc = run_decode(uocr, case)
    check_queries(case, [0, 1, 2], out, sel, sc)


@pytest.mark.slow
def test_chunked_prefill_workload_every_query_step_entries(uocr, cuda_device):
    """The chunked-prefill workload through the per-step entry points (scan, selection,
    query-centric attention): every score, selection and output of the 2048 queries."""
    case = workloads.chunked_prefill(device=cuda_device)
    sc = uocr.index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens, case.q_seq, case.q_pos)
    sel = uocr.block_topk(sc, case.seq_lens, case.q_seq, case.q_pos)
    out = uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, sel,
                           case.q_seq, case.q_pos)
    torch.cuda.synchronize()
    check_all_queries(case, out, sel, sc)
