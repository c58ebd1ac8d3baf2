"""uocr_sparse_decode_static: the decode call for callers that cannot allocate.

Some callers of this library cannot allocate device memory where they decode:
a plugin inside a host engine that owns every device allocation, or a decode
loop where a cudaMalloc (which may synchronise the device) is not allowed.
``uocr_sparse_decode_static`` serves them: the caller passes inputs and
outputs only, and the scratch lives in a fixed-size device array inside
libuocr.so.  These tests call it through the C ABI and compare it with
``uocr_sparse_decode`` on the same inputs, on two calls in a row with
different shapes (the second call reuses the array the first one left
behind), and check that oversized shapes are refused before any launch.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

OUT_MAX_ATOL = 2e-2
OUT_MEAN_ATOL = 2e-3


@pytest.fixture(scope="module")
def uocr(cuda_device):
    import block_sparse_long_uocr_b200 as m
    return m


def _both(uocr, case):
    ref_out, ref_sel = uocr.sparse_decode(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool,
                                          case.block_table, case.seq_lens)
    out = torch.full_like(case.q, float("nan"))
    sel = torch.full((case.n_q, 16), -7, dtype=torch.int32, device=case.q.device)
    before = torch.cuda.memory_allocated()
    uocr.sparse_decode_static(case.q, case.k_pool, case.v_pool, case.idx_q, case.idx_k_pool,
                              case.block_table, case.seq_lens, out=out, sel=sel)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before          # nothing allocated through torch either
    return ref_out, ref_sel, out, sel


def _assert_close(ref_out, ref_sel, out, sel):
    assert torch.equal(sel, ref_sel)
    d = (out.float() - ref_out.float()).abs()
    assert torch.isfinite(out.float()).all()
    assert d.max().item() <= OUT_MAX_ATOL and d.mean().item() <= OUT_MEAN_ATOL


def test_static_decode_matches_the_workspace_entry_on_two_calls_in_a_row(uocr, cuda_device):
    # first call: a ragged, shuffled batch
    a = workloads.make_case([32 * 900 + 7, 32 * 40, 129, 32 * 2000], shuffle=True, seed=31, device=cuda_device)
    _assert_close(*_both(uocr, a))
    # second call: other shapes and data; the shared scratch still holds the first call's contents
    b = workloads.make_case([32 * 3000, 5000, 64, 32 * 17 + 31, 32 * 1024, 100], shuffle=True, max_blocks=3200,
                            seed=32, device=cuda_device)
    _assert_close(*_both(uocr, b))
    # and the first case again, after the second has overwritten the scratch
    _assert_close(*_both(uocr, a))


def test_static_decode_refuses_shapes_beyond_its_scratch(uocr, cuda_device):
    B, H = 64, 10
    mb = 1
    while uocr.workspace_bytes(B, H, mb + 1) <= uocr.STATIC_SCRATCH_BYTES:   # the largest shape that fits
        mb += 1
    mb += 1                                         # one block more than the scratch holds
    assert uocr.workspace_bytes(B, H, mb) > uocr.STATIC_SCRATCH_BYTES >= uocr.workspace_bytes(B, H, mb - 1)
    q = torch.zeros((B, H, 128), dtype=torch.bfloat16, device=cuda_device)
    kv = torch.zeros((1, H, 32, 128), dtype=torch.bfloat16, device=cuda_device)
    ik = torch.zeros((1, 32, 128), dtype=torch.bfloat16, device=cuda_device)
    qi = torch.zeros((B, 128), dtype=torch.bfloat16, device=cuda_device)
    bt = torch.zeros((B, mb), dtype=torch.int32, device=cuda_device)
    sl = torch.ones((B,), dtype=torch.int32, device=cuda_device)
    out = torch.zeros_like(q)
    sel = torch.zeros((B, 16), dtype=torch.int32, device=cuda_device)
    with pytest.raises(uocr.UocrError) as e:
        uocr.sparse_decode_static(q, kv, kv, qi, ik, bt, sl, out=out, sel=sel)
    assert e.value.status == 3                      # UOCR_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out == 0).all() and (sel == 0).all()    # nothing was launched
