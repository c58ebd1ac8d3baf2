"""The comparator decode kernels (full causal attention; R-SWA-style reference
prefix plus the 128-token window) against the fp64 oracle's attention over the
same block set, through the C ABI."""
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


def comparator_blocks(nb, ref_blocks):
    return sorted(set(range(min(ref_blocks, nb))) | set(range(max(nb - 4, 0), nb)))


def check(case, out, ref_blocks):
    got = out.float().cpu().numpy()
    for b in range(case.n_q):
        p = int(case.q_pos[b])
        nb = p // 32 + 1 if p >= 0 else 0
        blocks = np.array(comparator_blocks(nb, ref_blocks), np.int32)
        ref = oracle.attend(case.q[b].cpu(), case.k_pool.cpu(), case.v_pool.cpu(), case.block_table[b].cpu(),
                            blocks if blocks.size else np.full(1, -1, np.int32), p)
        d = np.abs(got[b] - ref)
        assert d.max() <= 2e-2 and d.mean() <= 2e-3, (b, d.max(), d.mean())


@pytest.mark.parametrize("ref_blocks", [10 ** 6, 0, 7, 40])
def test_comparator_matches_oracle(uocr, cuda_device, ref_blocks):
    lens = [1, 31, 33, 128, 129, 600, 32 * 70 + 5, 32 * 100]
    case = workloads.make_case(lens, heads=3, shuffle=True, seed=ref_blocks % 97, device=cuda_device)
    out = uocr.dense_decode(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens,
                            ref_blocks=min(ref_blocks, case.max_blocks))
    torch.cuda.synchronize()
    check(case, out, ref_blocks)


def test_full_attention_equals_sparse_when_everything_fits(uocr, cuda_device):
    """With at most 16 causal blocks the sparse step attends to every block: same output."""
    case = workloads.make_case([100, 512, 17, 480], shuffle=True, seed=2, device=cuda_device)
    dense = uocr.dense_decode(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens)
    sparse, _ = uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool,
                                   case.block_table, case.seq_lens)
    torch.cuda.synchronize()
    assert (dense.float() - sparse.float()).abs().max().item() <= 1e-2


def test_comparator_long_context_sampled(uocr, cuda_device):
    case = workloads.long_decode(device=cuda_device, B=4, n_layers=1)
    out = uocr.dense_decode(case.q, case.k_pool, case.v_pool, case.block_table, case.seq_lens)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    b = 2
    nb = 4096
    pages = case.block_table[b, :nb].long()
    k = case.k_pool[pages].permute(1, 0, 2, 3).reshape(case.q.shape[1], -1, 128).double().cpu()
    v = case.v_pool[pages].permute(1, 0, 2, 3).reshape(case.q.shape[1], -1, 128).double().cpu()
    ref = torch.nn.functional.scaled_dot_product_attention(case.q[b].double().cpu().unsqueeze(1), k, v)
    d = np.abs(got[b] - ref.squeeze(1).numpy())
    assert d.max() <= 2e-2 and d.mean() <= 2e-3
