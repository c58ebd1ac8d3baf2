"""page2d rotary embedding + cache append (the step before the scan) against the
fp64 oracle, through the C ABI.  Outputs are bf16: each element must be within
one bf16 rounding (2^-8 relative) of the fp64 value, and every cache row other
than the new tokens' must be untouched."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def uocr(cuda_device):
    import block_sparse_long_uocr_b200 as m
    return m


def _close_bf16(got, want):
    got = got.float().cpu().double().numpy() if torch.is_tensor(got) else got
    err = np.abs(got - want)
    assert (err <= np.abs(want) * 2.0 ** -8 + 1e-6).all(), err.max()


def _run(uocr, cuda_device, lens, tok, page, q_seq=None, q_pos=None, seed=0, heads=10):
    case = workloads.make_case(lens, heads=heads, shuffle=True, seed=seed, device=cuda_device)
    n = len(tok)
    g = torch.Generator(device=cuda_device).manual_seed(seed + 1)
    q = torch.randn(n, heads, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    qi = torch.randn(n, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    kn = torch.randn(n, heads, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    vn = torch.randn(n, heads, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    kin = torch.randn(n, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    tp = torch.tensor(tok, dtype=torch.int32, device=cuda_device)
    pp = torch.tensor(page, dtype=torch.int32, device=cuda_device)
    qs = None if q_seq is None else torch.tensor(q_seq, dtype=torch.int32, device=cuda_device)
    qp = None if q_pos is None else torch.tensor(q_pos, dtype=torch.int32, device=cuda_device)
    seqs = np.arange(n) if q_seq is None else np.array(q_seq)
    pos = (case.seq_lens.cpu().numpy()[seqs] - 1) if q_pos is None else np.array(q_pos)
    want = oracle.rope_append(q, qi, kn, vn, kin, np.array(tok), np.array(page), seqs, pos, case.block_table,
                              case.k_pool, case.v_pool, case.idx_k_pool)
    kc, vc, ic = case.k_pool.clone(), case.v_pool.clone(), case.idx_k_pool.clone()
    q2, qi2 = q.clone(), qi.clone()
    uocr.rope_append(q2, qi2, kn, vn, kin, tp, pp, case.block_table, case.seq_lens, kc, vc, ic, qs, qp)
    torch.cuda.synchronize()
    return want, (q2, qi2, kc, vc, ic), case


@pytest.mark.parametrize("tok,page", [([0, 1, 2], [0, 1, 2]), ([37, 4095, 131071], [5, 0, 1000001]),
                                      ([900000, 12, 70000], [-3, 7, 2])])
def test_rope_append_decode_tokens(uocr, cuda_device, tok, page):
    lens = [100, 32 * 50, 32 * 7 + 31]
    want, got, case = _run(uocr, cuda_device, lens, tok, page, seed=tok[1] % 13)
    qr, qir, kc, vc, ic = want
    q2, qi2, kc2, vc2, ic2 = got
    _close_bf16(q2, qr)
    _close_bf16(qi2, qir)
    _close_bf16(kc2, kc)
    _close_bf16(ic2, ic)
    np.testing.assert_array_equal(vc2.float().cpu().double().numpy(), vc)     # values copied exactly


def test_rope_append_prefill_tokens(uocr, cuda_device):
    """A chunk of new tokens of one sequence at explicit positions (rows of several pages)."""
    n = 70
    pos = list(range(1000 - n, 1000))
    tok = [p % 517 for p in pos]
    page = [p // 517 for p in pos]
    want, got, case = _run(uocr, cuda_device, [1000], tok, page, q_seq=[0] * n, q_pos=pos, seed=3, heads=2)
    for w, g in zip(want[:2] + want[2:3] + want[4:5], got[:2] + got[2:3] + got[4:5]):
        _close_bf16(g, w)
    np.testing.assert_array_equal(got[3].float().cpu().double().numpy(), want[3])


def test_rope_append_skips_and_flags_bad_rows(uocr, cuda_device):
    case = workloads.make_case([64, 64], heads=2, seed=4, device=cuda_device)
    bt = case.block_table.clone()
    bt[1, 1] = case.num_pages + 9            # the second sequence's new token lands on a bad page
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device=cuda_device)
    q, qi, kn, vn, kin = z(2, 2, 128), z(2, 128), torch.ones(2, 2, 128, dtype=torch.bfloat16, device=cuda_device), \
        torch.ones(2, 2, 128, dtype=torch.bfloat16, device=cuda_device), z(2, 128)
    kc = case.k_pool.clone()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    i32 = lambda v: torch.tensor(v, dtype=torch.int32, device=cuda_device)
    uocr.rope_append(q, qi, kn, vn, kin, i32([0, 0]), i32([0, 0]), bt, case.seq_lens, kc, case.v_pool.clone(),
                     case.idx_k_pool.clone(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & uocr.DEVERR_PAGE
    page0 = int(case.block_table[0, 1])
    assert (kc[page0, :, 31] == 1).all()                     # the good token was written (identity rotation)
    changed = (kc != case.k_pool).any(dim=(1, 2, 3)).nonzero().flatten().tolist()
    assert changed == [page0]
