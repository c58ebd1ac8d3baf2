"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before launching anything.

These run without a GPU.  Calls with fake pointers are made only on hosts
with no CUDA device, and every one of them carries an argument that the host
validation rejects before any CUDA call.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "uocr.h")


@pytest.fixture(scope="module")
def pkg():
    from block_sparse_long_uocr_b200 import build
    build.build()
    import block_sparse_long_uocr_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(uocr_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["uocr_index_score", "uocr_block_topk", "uocr_sparse_attn", "uocr_sparse_decode",
              "uocr_workspace_bytes", "uocr_status_string", "uocr_abi_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(pkg):
    out = subprocess.run(["nm", "-D", "--defined-only", pkg.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (uocr_[a-z0-9_]+)\b", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(pkg.lib, n)


def test_status_strings_and_version(pkg):
    for code in range(5):
        s = pkg.lib.uocr_status_string(code).decode()
        assert s.startswith(pkg.STATUS[code])
    assert pkg.lib.uocr_status_string(99).decode() == "UOCR_ERR_UNKNOWN"
    assert pkg.lib.uocr_abi_version() == 2


def test_last_cuda_error_names_no_error_before_any_failure(pkg):
    # host-side rejections return before any CUDA call, so they leave no CUDA error behind
    assert pkg.lib.uocr_last_cuda_error().decode() == "no error"


def test_workspace_is_a_pure_function_of_shapes(pkg):
    ws = pkg.workspace_bytes
    assert ws(0, 10, 64) == 0 and ws(4, 0, 64) == 0 and ws(4, 10, 0) == 0
    a = ws(16, 10, 4096)
    assert a == ws(16, 10, 4096) and a % 256 == 0
    assert a == 16 * 4096 * 4                       # the block-score scratch, nothing else
    assert ws(32, 10, 4096) > a and ws(16, 10, 8192) > a
    assert ws(16, 1, 4096) == a                     # heads do not change it (attention merges on chip)
    assert ws(3, 10, 5) == 256                      # rounded up to 256 bytes


# --------------------------------------------------------------------------- host fault injection
no_gpu = pytest.mark.skipif(torch.cuda.is_available(),
                            reason="fake-pointer calls run only on hosts without a CUDA device")
FAKE = 1 << 20          # 16-byte aligned, never dereferenced: every call below fails validation first
MIS = FAKE + 2          # misaligned for bf16 / int32


def _score_args(**over):
    a = dict(idx_q=FAKE, idx_k=FAKE, bt=FAKE, sl=FAKE, qs=None, qp=None, n_q=4, B=4, mb=64, P=256,
             scores=FAKE, err=None)
    a.update(over)
    return a


def _call_score(lib, a):
    return lib.uocr_index_score(a["idx_q"], a["idx_k"], a["bt"], a["sl"], a["qs"], a["qp"], a["n_q"], a["B"],
                                a["mb"], a["P"], a["scores"], a["err"], None)


@no_gpu
@pytest.mark.parametrize("over", [dict(idx_q=None), dict(idx_k=None), dict(bt=None), dict(sl=None),
                                  dict(scores=None), dict(n_q=-1), dict(B=0), dict(mb=0), dict(P=0),
                                  dict(idx_q=MIS), dict(idx_k=FAKE + 8), dict(bt=MIS), dict(scores=MIS),
                                  dict(qs=MIS), dict(qp=MIS), dict(err=MIS)])
def test_index_score_rejects(pkg, over):
    assert _call_score(pkg.lib, _score_args(**over)) == 1


@no_gpu
def test_index_score_rejects_huge_block_count(pkg):
    assert _call_score(pkg.lib, _score_args(mb=1 << 27)) == 2


@no_gpu
def test_zero_queries_is_a_no_op(pkg):
    # n_q == 0 returns before touching the device
    assert _call_score(pkg.lib, _score_args(n_q=0)) == 0
    assert pkg.lib.uocr_block_topk(FAKE, FAKE, None, None, 0, 4, 64, FAKE, None, None) == 0


@no_gpu
@pytest.mark.parametrize("args", [
    (None, FAKE, None, None, 4, 4, 64, FAKE),     # scores NULL
    (FAKE, None, None, None, 4, 4, 64, FAKE),     # seq_lens NULL
    (FAKE, FAKE, None, None, 4, 4, 64, None),     # sel NULL
    (FAKE, FAKE, None, None, 4, 0, 64, FAKE),     # B < 1
    (FAKE, FAKE, None, None, 4, 4, 0, FAKE),      # max_blocks < 1
    (MIS, FAKE, None, None, 4, 4, 64, FAKE),      # misaligned scores
    (FAKE, FAKE, None, None, 4, 4, 64, MIS),      # misaligned sel
])
def test_block_topk_rejects(pkg, args):
    assert pkg.lib.uocr_block_topk(*args, None, None) == 1


def _call_attn(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, sel=FAKE, n_q=4, B=4, H=10, mb=64, P=256,
             scale=0.088, out=FAKE)
    a.update(over)
    return lib.uocr_sparse_attn(a["q"], a["k"], a["v"], a["bt"], a["sl"], None, None, a["sel"], a["n_q"],
                                a["B"], a["H"], a["mb"], a["P"], ctypes.c_float(a["scale"]), a["out"], None, None)


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(k=MIS), 1), (dict(v=None), 1), (dict(out=FAKE + 4), 1), (dict(sel=None), 1),
    (dict(H=0), 2), (dict(H=65), 2), (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1),
    (dict(sel=MIS), 1), (dict(bt=None), 1), (dict(P=0), 1),
])
def test_sparse_attn_rejects(pkg, over, code):
    assert _call_attn(pkg.lib, **over) == code


@no_gpu
def test_sparse_decode_workspace_boundary(pkg):
    need = pkg.workspace_bytes(4, 10, 64)
    a = [FAKE] * 7 + [4, 10, 64, 256, FAKE, FAKE, FAKE]
    assert pkg.lib.uocr_sparse_decode(*a, need - 1, None, None) == 3
    assert pkg.lib.uocr_sparse_decode(*a[:13], FAKE + 128, need, None, None) == 3   # misaligned workspace


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(sel=None), 1), (dict(idx_q=None), 1), (dict(idx_k=MIS), 1), (dict(H=0), 2),
    (dict(wsb=0), 3), (dict(ws=None), 3), (dict(B=0), 1), (dict(mb=0), 1),
])
def test_sparse_decode_rejects(pkg, over, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, idx_q=FAKE, idx_k=FAKE, bt=FAKE, sl=FAKE, B=4, H=10, mb=64, P=256,
             out=FAKE, sel=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(over)
    st = pkg.lib.uocr_sparse_decode(a["q"], a["k"], a["v"], a["idx_q"], a["idx_k"], a["bt"], a["sl"], a["B"],
                                    a["H"], a["mb"], a["P"], a["out"], a["sel"], a["ws"], a["wsb"], None, None)
    assert st == code


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(sel=None), 1), (dict(idx_k=MIS), 1), (dict(H=0), 2), (dict(B=0), 1),
    (dict(mb=1 << 27), 2),                               # too many blocks: UNSUPPORTED, not WORKSPACE
    (dict(q=None, B=64, mb=1 << 20), 1),                 # a NULL pointer with a shape past the scratch
    (dict(P=0, B=64, mb=1 << 20), 1),                    # a bad pool size with a shape past the scratch
    (dict(B=64, mb=1 << 20), 3),                         # valid arguments, scratch too small
])
def test_sparse_decode_static_checks_in_the_order_of_sparse_decode(pkg, over, code):
    """The static entry returns what uocr_sparse_decode would for the same arguments; only a call
    that passes all of those checks can fail on its fixed scratch size (UOCR_ERR_WORKSPACE)."""
    a = dict(q=FAKE, k=FAKE, v=FAKE, idx_q=FAKE, idx_k=FAKE, bt=FAKE, sl=FAKE, B=4, H=10, mb=64, P=256,
             out=FAKE, sel=FAKE)
    a.update(over)
    st = pkg.lib.uocr_sparse_decode_static(a["q"], a["k"], a["v"], a["idx_q"], a["idx_k"], a["bt"], a["sl"],
                                           a["B"], a["H"], a["mb"], a["P"], a["out"], a["sel"], None, None)
    assert st == code
    if code != 3:
        ws = pkg.workspace_bytes(a["B"], a["H"], a["mb"]) if a["B"] > 0 and a["H"] > 0 and a["mb"] > 0 else 0
        st2 = pkg.lib.uocr_sparse_decode(a["q"], a["k"], a["v"], a["idx_q"], a["idx_k"], a["bt"], a["sl"], a["B"],
                                         a["H"], a["mb"], a["P"], a["out"], a["sel"], FAKE, max(ws, 256), None, None)
        assert st2 == code


def test_python_binding_refuses_cpu_tensors(pkg):
    x = torch.zeros(2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pkg.index_score(x, torch.zeros(4, 32, 128, dtype=torch.bfloat16), torch.zeros(2, 4, dtype=torch.int32),
                        torch.ones(2, dtype=torch.int32))


def test_product_package_does_not_import_the_oracle():
    pkg_dir = os.path.join(ROOT, "block_sparse_long_uocr_b200")
    for dirpath, _, files in os.walk(pkg_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\boracle\b", src.replace("oracle-free", "")), f"{f} mentions the oracle"


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q_pos=None), 1), (dict(seq=-1), 1), (dict(seq=4), 1), (dict(idx_q=MIS), 1), (dict(scores=None), 1),
    (dict(B=0), 1), (dict(mb=0), 1), (dict(P=0), 1), (dict(idx_k=None), 1),
])
def test_prefill_index_score_rejects(pkg, over, code):
    a = dict(idx_q=FAKE, idx_k=FAKE, bt=FAKE, sl=FAKE, seq=0, q_pos=FAKE, n_q=4, B=4, mb=64, P=256, scores=FAKE)
    a.update(over)
    st = pkg.lib.uocr_prefill_index_score(a["idx_q"], a["idx_k"], a["bt"], a["sl"], a["seq"], a["q_pos"], a["n_q"],
                                          a["B"], a["mb"], a["P"], a["scores"], None, None)
    assert st == code


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q_pos=None), 1), (dict(seq=5), 1), (dict(sel=None), 1), (dict(out=MIS), 1), (dict(H=0), 2),
    (dict(ws=None), 3), (dict(wsb=16), 3), (dict(ws=FAKE + 64), 3),
])
def test_sparse_prefill_rejects(pkg, over, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, idx_q=FAKE, idx_k=FAKE, bt=FAKE, sl=FAKE, seq=0, q_pos=FAKE, n_q=4, B=4, H=10,
             mb=64, P=256, out=FAKE, sel=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(over)
    st = pkg.lib.uocr_sparse_prefill(a["q"], a["k"], a["v"], a["idx_q"], a["idx_k"], a["bt"], a["sl"], a["seq"],
                                     a["q_pos"], a["n_q"], a["B"], a["H"], a["mb"], a["P"], a["out"], a["sel"],
                                     a["ws"], a["wsb"], None, None)
    assert st == code


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q_pos=None), 1), (dict(seq=5), 1), (dict(seq=-1), 1), (dict(sel=None), 1), (dict(sel=MIS), 1),
    (dict(out=MIS), 1), (dict(q=None), 1), (dict(H=0), 2), (dict(H=65), 2), (dict(scale=float("nan")), 1),
    (dict(ws=None), 3), (dict(wsb=16), 3), (dict(ws=FAKE + 64), 3), (dict(mb=0), 1), (dict(P=0), 1),
])
def test_sparse_attn_seq_rejects(pkg, over, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, seq=0, q_pos=FAKE, sel=FAKE, n_q=4, B=4, H=10, mb=64, P=256,
             scale=0.088, out=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(over)
    st = pkg.lib.uocr_sparse_attn_seq(a["q"], a["k"], a["v"], a["bt"], a["sl"], a["seq"], a["q_pos"], a["sel"],
                                      a["n_q"], a["B"], a["H"], a["mb"], a["P"], a["scale"], a["out"], a["ws"],
                                      a["wsb"], None, None)
    assert st == code


def test_sparse_attn_seq_workspace_is_a_pure_function_of_shapes(pkg):
    f = pkg.sparse_attn_seq_workspace_bytes
    assert f(0, 10, 64) == 0 and f(4, 0, 64) == 0 and f(4, 10, 0) == 0
    a = f(2048, 10, 2048)
    assert a == f(2048, 10, 2048) and a % 256 == 0
    # the inversion (counts, list counters, items, entries, the checked selection) and the partial states
    assert a >= 2048 * 10 * 16 * (128 * 2 + 8) + 2048 * 16 * (8 + 4) + 2 * 2048 * 4
    assert f(2048, 1, 2048) < a and f(4096, 10, 2048) > a


def test_prefill_workspace_is_a_pure_function_of_shapes(pkg):
    pw, ws = pkg.prefill_workspace_bytes, pkg.workspace_bytes
    assert pw(0, 10, 64) == 0 and pw(4, 0, 64) == 0 and pw(4, 10, 0) == 0
    a = pw(2048, 10, 2048)
    assert a == pw(2048, 10, 2048) and a % 256 == 0
    # scores, then the inverted index (2 x max_blocks ints, 16 n_q (entry, position) pairs, the item
    # records) and 16 partial states per (query, head): 128 bf16 outputs + fp32 (m, l)
    assert a >= ws(2048, 10, 2048) + 2048 * 10 * 16 * (128 * 2 + 8) + 2048 * 16 * 8 + 2 * 2048 * 4
    assert pw(2048, 1, 2048) < a and pw(4096, 10, 2048) > a
