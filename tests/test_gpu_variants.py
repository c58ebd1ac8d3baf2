"""The selection variants of the next-step rows, against the fp64 oracle through the C ABI:
block-summary scoring (one summary vector per block; the mean-key summary builder; the
decode step built on it) and selection under a page-aware candidate mask."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import accept_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def uocr(cuda_device):
    import block_sparse_long_uocr_b200 as m
    return m


def _summaries(num_pages, device, seed):
    g = torch.Generator(device=device).manual_seed(seed)
    return torch.randn(num_pages, 128, generator=g, device=device).to(torch.bfloat16)


def test_summary_scores_match_oracle(uocr, cuda_device):
    lens = [1, 31, 129, 32 * 300 + 7, 5000]
    case = workloads.make_case(lens, heads=1, shuffle=True, seed=6, device=cuda_device)
    summ = _summaries(case.num_pages, cuda_device, 7)
    sc = uocr.summary_score(case.idx_q, summ, case.block_table, case.seq_lens)
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        want = oracle.summary_scores(case.idx_q[b], summ, case.block_table[b], L - 1)
        np.testing.assert_allclose(sc[b, : want.shape[0]].cpu().double().numpy(), want, rtol=0, atol=1e-3)
        assert torch.isneginf(sc[b, want.shape[0]:]).all()


def test_block_summary_mean_matches_oracle(uocr, cuda_device):
    case = workloads.make_case([32 * 40], heads=1, shuffle=True, seed=8, device=cuda_device)
    summ = uocr.block_summary_mean(case.idx_k_pool)
    pages = torch.tensor([3, 0, 39], dtype=torch.int32, device=cuda_device)
    partial = torch.zeros_like(summ)
    uocr.block_summary_mean(case.idx_k_pool, partial, pages)
    torch.cuda.synchronize()
    for page in range(case.num_pages):
        want = oracle.block_mean(case.idx_k_pool, page)
        err = np.abs(summ[page].float().cpu().double().numpy() - want)
        assert (err <= np.abs(want) * 2.0 ** -8 + 1e-6).all()
    touched = (partial != 0).any(dim=1).nonzero().flatten().tolist()
    assert touched == [0, 3, 39] and torch.equal(partial[3], summ[3])


def test_sparse_decode_summary_matches_oracle(uocr, cuda_device):
    lens = [40, 32 * 100, 32 * 700 + 9, 32 * 2000]
    case = workloads.make_case(lens, shuffle=True, seed=9, device=cuda_device)
    summ = _summaries(case.num_pages, cuda_device, 10)
    out, sel = uocr.sparse_decode_summary(case.q, case.k_pool, case.v_pool, case.idx_q, summ, case.block_table,
                                          case.seq_lens)
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        s = oracle.summary_scores(case.idx_q[b], summ, case.block_table[b], L - 1)
        want_sel, tie = oracle.select(s, s.shape[0])
        got_sel = sel[b].cpu().numpy()
        assert accept_selection(s, want_sel, got_sel, tie)
        pages = case.block_table[b, torch.tensor([j for j in got_sel if j >= 0])].long()
        bt = np.full(case.max_blocks, -1, np.int32)
        for n, j in enumerate([j for j in got_sel if j >= 0]):
            bt[j] = n
        ref = oracle.attend(case.q[b], case.k_pool[pages], case.v_pool[pages], bt, got_sel, L - 1)
        d = np.abs(out[b].float().cpu().numpy() - ref)
        assert d.max() <= 2e-2 and d.mean() <= 2e-3


def _random_mask(B, max_blocks, density, seed):
    rng = np.random.default_rng(seed)
    words = (max_blocks + 31) // 32
    bits = rng.random((B, words * 32)) < density
    m = np.zeros((B, words), np.uint32)
    for w in range(words):
        for k in range(32):
            m[:, w] |= (bits[:, w * 32 + k].astype(np.uint32) << np.uint32(k))
    return m


@pytest.mark.parametrize("mb", [4096, 4093])
@pytest.mark.parametrize("density,kind", [(0.5, "normal"), (0.05, "normal"), (0.005, "ties"), (1.0, "ties"),
                                          (0.3, "ties"), (0.0, "normal")])
def test_masked_topk_is_exact(uocr, cuda_device, density, kind, mb):
    """Few rows (one CTA per row, keys in registers); an odd row length starts rows off a
    16-byte boundary (scalar reads)."""
    g = torch.Generator().manual_seed(int(density * 1000) + len(kind) + mb)
    lens = [min(L, 32 * mb) for L in (1, 100, 128, 129, 545, 32 * 1024, 32 * 4096, 77777)]
    s = torch.randint(-4, 5, (len(lens), mb), generator=g).float() if kind == "ties" else \
        torch.randn(len(lens), mb, generator=g)
    mask = _random_mask(len(lens), mb, density, seed=len(lens))
    sel = uocr.block_topk_masked(s.to(cuda_device), torch.tensor(lens, dtype=torch.int32, device=cuda_device),
                                 torch.from_numpy(mask.view(np.int32)).to(cuda_device))
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        nb = (L - 1) // 32 + 1
        want, _ = oracle.select_masked(s[b].double().numpy(), nb, mask[b])
        assert sel[b].cpu().tolist() == want.tolist(), (b, nb)


@pytest.mark.parametrize("density,kind", [(0.5, "normal"), (0.01, "ties"), (1.0, "ties")])
def test_masked_topk_many_rows_is_exact(uocr, cuda_device, density, kind):
    """The warp-per-row selection (many rows) under a candidate mask."""
    g = torch.Generator().manual_seed(int(density * 100) + 7)
    n, mb = 600, 1024
    lens = [1, 100, 128, 129, 545, 32 * mb] + torch.randint(1, 32 * mb + 1, (n - 6,), generator=g).tolist()
    s = torch.randint(-4, 5, (n, mb), generator=g).float() if kind == "ties" else torch.randn(n, mb, generator=g)
    mask = _random_mask(n, mb, density, seed=n)
    sel = uocr.block_topk_masked(s.to(cuda_device), torch.tensor(lens, dtype=torch.int32, device=cuda_device),
                                 torch.from_numpy(mask.view(np.int32)).to(cuda_device)).cpu()
    for b, L in enumerate(lens):
        nb = (L - 1) // 32 + 1
        want, _ = oracle.select_masked(s[b].double().numpy(), nb, mask[b])
        assert sel[b].tolist() == want.tolist(), (b, nb)


def test_masked_selection_end_to_end(uocr, cuda_device):
    lens = [32 * 300, 32 * 64 + 5, 32 * 900]
    case = workloads.make_case(lens, shuffle=True, seed=12, device=cuda_device)
    mask = _random_mask(3, case.max_blocks, 0.2, seed=13)
    sc = uocr.index_score(case.idx_q, case.idx_k_pool, case.block_table, case.seq_lens)
    sel = uocr.block_topk_masked(sc, case.seq_lens, torch.from_numpy(mask.view(np.int32)).to(cuda_device))
    out = uocr.sparse_attn(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens, sel)
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        s = oracle.block_scores(case.idx_q[b], case.idx_k_pool, case.block_table[b], L - 1)
        want, tie = oracle.select_masked(s, s.shape[0], mask[b])
        assert not tie and sel[b].cpu().tolist() == want.tolist()
        for j in want[:12]:
            if 0 <= j < s.shape[0] - 4:
                assert (mask[b][j // 32] >> (j % 32)) & 1
        ref = oracle.attend(case.q[b], case.k_pool, case.v_pool, case.block_table[b], want, L - 1)
        d = np.abs(out[b].float().cpu().numpy() - ref)
        assert d.max() <= 2e-2 and d.mean() <= 2e-3
