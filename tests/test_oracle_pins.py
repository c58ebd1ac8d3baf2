"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test fixes one part of the oracle with something independent of its code:
closed forms on constructed inputs, brute-force enumeration on tiny inputs,
invariants the method must satisfy, a library attention routine
(torch scaled_dot_product_attention in fp64) in the cases where the sparse
step reduces to dense causal attention, and the constants the pages print
(tests/golden/page_constants.json).  A plausible slip in the oracle (a dropped
causal mask, a wrong tie order, a transposed page layout, a missing scale, a
local block leaking into the remote slots) fails at least one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")


def bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


# ----------------------------------------------------------------------------- page constants
def test_page_constants_match_oracle():
    g = json.load(open(GOLDEN))
    assert oracle.BLOCK == g["sparse_block_size"]["value"]
    assert oracle.N_LOCAL == g["sparse_local_block"]["value"]
    assert oracle.N_REMOTE == g["dash_topk_blocks"]["value"]
    assert oracle.N_SEL == g["sparse_topk_blocks"]["value"]
    assert oracle.N_LOCAL * oracle.BLOCK == g["sliding_window_size"]["value"]
    assert oracle.N_SEL * oracle.BLOCK == g["read_set_tokens"]["value"]
    assert oracle.HEADS == g["num_attention_heads"]["value"]
    assert oracle.HEAD_DIM == g["head_dim"]["value"]
    assert oracle.IDX_DIM == g["indexer_dim"]["value"]
    frac = g["read_set_tokens"]["value"] / g["read_fraction_at_128k_below"]["context"]
    assert frac < g["read_fraction_at_128k_below"]["value"]
    # K and V, bf16, all layers at 128K: same order as the page's estimate (within 10 %).
    kv = g["num_layers"]["value"] * 131072 * oracle.HEADS * oracle.HEAD_DIM * 2 * 2 / 1e9
    assert abs(kv - g["kv_cache_128k_gb_estimate"]["value"]) / kv < 0.10


# ----------------------------------------------------------------------------- block scores
def _ramp_case(n_blocks, sign=1.0, d_idx=128):
    """idx_q = e_0, idx_k[t][0] = sign * t/64 (exact in bf16 for t < 256), everything else 0."""
    qi = torch.zeros(d_idx)
    qi[0] = 1.0
    ki = torch.zeros(n_blocks * 32, d_idx)
    ki[:, 0] = sign * torch.arange(n_blocks * 32, dtype=torch.float32) / 64.0
    assert torch.equal(bf16(ki).float(), ki)
    return bf16(qi), bf16(ki).view(n_blocks, 32, d_idx)


@pytest.mark.parametrize("p", [255, 200, 31, 0, 32, 100])
def test_scores_closed_form_increasing(p):
    qi, pages = _ramp_case(8)
    s = oracle.block_scores(qi, pages, np.arange(8), p)
    nb = p // 32 + 1
    want = [min(32 * j + 31, p) / 64.0 for j in range(nb)]
    assert s.shape == (nb,)
    assert s.tolist() == want


def test_scores_closed_form_decreasing():
    qi, pages = _ramp_case(8, sign=-1.0)
    s = oracle.block_scores(qi, pages, np.arange(8), 255)
    assert s.tolist() == [-(32 * j) / 64.0 for j in range(8)]


def test_scores_use_the_block_table():
    qi, pages = _ramp_case(8)
    perm = np.array([5, 2, 7, 0, 1, 6, 3, 4])
    shuffled = torch.empty_like(pages)
    shuffled[perm] = pages                    # logical block j lives at physical page perm[j]
    s = oracle.block_scores(qi, shuffled, perm, 255)
    assert s.tolist() == [(32 * j + 31) / 64.0 for j in range(8)]


def test_scores_brute_force_random():
    g = torch.Generator().manual_seed(7)
    qi = bf16(torch.randn(128, generator=g))
    pages = bf16(torch.randn(5, 32, 128, generator=g))
    for p in [0, 17, 63, 64, 159]:
        s = oracle.block_scores(qi, pages, np.arange(5), p)
        dots = pages.double().reshape(-1, 128)[: p + 1] @ qi.double()
        want = [dots[32 * j: 32 * j + 32].max().item() for j in range((p // 32) + 1)]
        np.testing.assert_allclose(s, want, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- selection
def _brute_force_select(s, nb, n_local, n_remote):
    """All subsets of the remote candidates of size min(n_remote, n_cand); keep the
    maximum-sum ones; the chosen one is the lexicographically smallest of them."""
    n_cand = max(nb - n_local, 0)
    k = min(n_remote, n_cand)
    best, best_sets = None, []
    for comb in itertools.combinations(range(n_cand), k):
        tot = sum(s[j] for j in comb)
        if best is None or tot > best:
            best, best_sets = tot, [comb]
        elif tot == best:
            best_sets.append(comb)
    chosen = sorted(min(best_sets)) + list(range(max(nb - n_local, 0), nb))
    return sorted(chosen), len(best_sets)


@pytest.mark.parametrize("seed", range(40))
def test_select_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(0, 13))
    n_local = int(rng.integers(0, 5))
    n_remote = int(rng.integers(0, 6))
    s = rng.integers(-3, 4, size=max(nb, 1)).astype(np.float64)  # small integers: exact sums, many ties
    sel, tie = oracle.select(s, nb, n_local, n_remote, tie_eps=0.5)
    want, n_opt = _brute_force_select(s, nb, n_local, n_remote)
    assert sel.tolist() == want + [-1] * (n_local + n_remote - len(want))
    # With integer scores and eps = 0.5 the near-tie flag means "more than one optimal set".
    n_cand = max(nb - n_local, 0)
    assert tie == (n_cand > n_remote and n_opt > 1)


def test_select_small_context_takes_everything():
    for nb in range(0, 17):
        sel, tie = oracle.select(np.random.default_rng(nb).standard_normal(max(nb, 1)), nb)
        assert sel.tolist() == list(range(nb)) + [-1] * (16 - nb)
        assert not tie


def test_select_remote_never_in_local_window():
    rng = np.random.default_rng(3)
    for nb in [17, 40, 100]:
        s = rng.standard_normal(nb)
        s[nb - 4:] = 1e9                      # local blocks score highest: they still take no remote slot
        sel, _ = oracle.select(s, nb)
        assert list(sel[-4:]) == list(range(nb - 4, nb))
        remote = sel[:12]
        assert (remote < nb - 4).all() and len(set(remote.tolist())) == 12
        top = np.argsort(-s[: nb - 4], kind="stable")[:12]
        assert sorted(top.tolist()) == remote.tolist()


def _oracle_sel(case, **kw):
    return oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool,
                      case.block_table, case.q_seq, case.q_pos, want_out=False, **kw)


def test_local_window_invariant_on_keys():
    """Whatever the local blocks' indexer keys hold, they are selected and the remote set does not move."""
    case = workloads.make_case([32 * 40 - 5, 32 * 21], heads=1, seed=11)
    base = _oracle_sel(case)["sel"]
    for fill in (+40.0, -40.0):
        ikp = case.idx_k_pool.clone()
        for b in range(2):
            nb = (int(case.seq_lens[b]) + 31) // 32
            for j in range(nb - 4, nb):
                page = int(case.block_table[b, j])
                ikp[page] = bf16(fill * case.idx_q[b].float()).expand(32, -1)
        alt = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, ikp, case.block_table,
                         case.q_seq, case.q_pos, want_out=False)["sel"]
        assert np.array_equal(base, alt)


def test_planted_references_are_recovered():
    case = workloads.make_case([32768, 32768, 32 * 300], heads=1, planted_blocks=12, seed=0)
    r = _oracle_sel(case)
    for b in range(3):
        nb = (int(case.seq_lens[b]) + 31) // 32
        assert sorted(case.planted[b]) == r["sel"][b, :12].tolist()
        assert r["sel"][b, 12:].tolist() == list(range(nb - 4, nb))
        assert not r["near_tie"][b]


def test_selection_is_scale_invariant():
    case = workloads.make_case([32 * 64, 32 * 50 + 7], heads=1, seed=5)
    base = _oracle_sel(case)["sel"]
    doubled = (case.idx_q.float() * 2).to(torch.bfloat16)   # exact in bf16
    alt = oracle.run(case.q, doubled, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                     case.q_seq, case.q_pos, want_out=False)["sel"]
    assert np.array_equal(base, alt)


# ----------------------------------------------------------------------------- attention
def _dense_sdpa(case, b, p):
    """Dense causal attention of the query at p over tokens 0..p (torch SDPA, fp64, CPU)."""
    nb = p // 32 + 1
    pages = case.block_table[b, :nb].long()
    k = case.k_pool[pages].double().permute(1, 0, 2, 3).reshape(case.k_pool.shape[1], -1, 128)[:, : p + 1]
    v = case.v_pool[pages].double().permute(1, 0, 2, 3).reshape(case.v_pool.shape[1], -1, 128)[:, : p + 1]
    qi = [i for i in range(case.n_q) if int(case.q_seq[i]) == b and int(case.q_pos[i]) == p][0]
    q = case.q[qi].double().unsqueeze(1)                     # [H, 1, D]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v).squeeze(1).numpy()


def test_dense_equivalence_when_everything_fits():
    """With at most 16 causal blocks every block is selected: the step is dense causal attention."""
    lens = [1, 31, 32, 33, 200, 512]
    case = workloads.make_case(lens, heads=3, shuffle=True, seed=2)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(r["out"][b], _dense_sdpa(case, b, L - 1), rtol=0, atol=1e-12)


def test_dense_equivalence_with_wide_topk_and_prefill_positions():
    """Parametrised oracle: n_remote >= candidates reduces to dense causal attention at any p."""
    case = workloads.make_case([32 * 30], heads=2, q_seq=[0] * 5, q_pos=[0, 45, 511, 700, 959], seed=4)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos, n_remote=40)
    for i, p in enumerate([0, 45, 511, 700, 959]):
        np.testing.assert_allclose(r["out"][i], _dense_sdpa(case, 0, p), rtol=0, atol=1e-12)


def test_sparse_differs_from_dense_on_long_context():
    """Sanity: with 40 blocks the 16-block selection is not dense attention (the mask matters)."""
    case = workloads.make_case([32 * 40], heads=2, seed=4)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    assert np.abs(r["out"][0] - _dense_sdpa(case, 0, 32 * 40 - 1)).max() > 1e-3


def test_constant_values_give_constant_output():
    case = workloads.make_case([32 * 30 + 9], heads=2, seed=8)
    v = torch.full_like(case.v_pool, 0.0)
    v[..., :] = bf16(torch.linspace(-2, 2, 128))
    r = oracle.run(case.q, case.idx_q, case.k_pool, v, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    np.testing.assert_allclose(r["out"][0], np.broadcast_to(bf16(torch.linspace(-2, 2, 128)).double().numpy(), (2, 128)),
                               rtol=0, atol=1e-12)


def test_zero_query_gives_mean_of_selected_values():
    case = workloads.make_case([32 * 30 + 9], heads=2, seed=9)
    q0 = torch.zeros_like(case.q)
    r = oracle.run(q0, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    p = int(case.q_pos[0])
    rows = []
    for j in r["sel"][0]:
        if j < 0:
            continue
        page = int(case.block_table[0, j])
        n = min(32, p + 1 - 32 * j)
        rows.append(case.v_pool[page, :, :n].double())
    mean = torch.cat(rows, dim=1).mean(dim=1).numpy()
    np.testing.assert_allclose(r["out"][0], mean, rtol=0, atol=1e-12)


def test_output_is_a_convex_combination():
    case = workloads.make_case([32 * 50 + 3, 32 * 19], heads=3, seed=10)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    vmin = case.v_pool.float().amin(dim=(0, 2)).double().numpy()
    vmax = case.v_pool.float().amax(dim=(0, 2)).double().numpy()
    assert (r["out"] >= vmin - 1e-12).all() and (r["out"] <= vmax + 1e-12).all()


def test_scale_argument_is_applied():
    """scale -> 0 turns the softmax uniform: the output becomes the mean of the selected values."""
    case = workloads.make_case([32 * 20], heads=1, seed=12)
    r0 = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                    case.q_seq, case.q_pos, scale=0.0)
    rq = oracle.run(torch.zeros_like(case.q), case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool,
                    case.block_table, case.q_seq, case.q_pos)
    np.testing.assert_allclose(r0["out"], rq["out"], rtol=0, atol=1e-14)
    r1 = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                    case.q_seq, case.q_pos)
    assert np.abs(r1["out"] - r0["out"]).max() > 1e-2


def test_paging_invariance():
    lens = [32 * 70 + 5, 32 * 33, 32 * 18 + 31]
    a = workloads.make_case(lens, heads=2, shuffle=False, seed=21)
    # same logical content, pages scattered over the pool in another order
    perm = torch.randperm(a.num_pages, generator=torch.Generator().manual_seed(99))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(a.num_pages)
    kp, vp, ikp = (torch.empty_like(t) for t in (a.k_pool, a.v_pool, a.idx_k_pool))
    kp[inv], vp[inv], ikp[inv] = a.k_pool, a.v_pool, a.idx_k_pool
    bt = a.block_table.clone()
    valid = bt >= 0
    bt[valid] = inv[bt[valid].long()].to(torch.int32)
    ra = oracle.run(a.q, a.idx_q, a.k_pool, a.v_pool, a.idx_k_pool, a.block_table, a.q_seq, a.q_pos)
    rb = oracle.run(a.q, a.idx_q, kp, vp, ikp, bt, a.q_seq, a.q_pos)
    assert np.array_equal(ra["sel"], rb["sel"])
    assert np.array_equal(ra["out"], rb["out"])
    assert np.array_equal(ra["scores"], rb["scores"])


def test_attention_over_given_selection_matches_attend():
    case = workloads.make_case([32 * 40 + 1], heads=2, seed=13)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, case.q_pos)
    other = np.array([[0, 3, 5, 7, 9, 11, 13, 15, 17, 19, 21, 23, 37, 38, 39, 40]], dtype=np.int32)
    r2 = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                    case.q_seq, case.q_pos, sel_in=other)
    direct = oracle.attend(case.q[0], case.k_pool, case.v_pool, case.block_table[0], other[0], int(case.q_pos[0]))
    np.testing.assert_array_equal(r2["out"][0], direct)
    assert np.abs(r2["out"][0] - r["out"][0]).max() > 1e-3


def test_empty_query_gives_zero_output():
    case = workloads.make_case([32], heads=1, seed=1)
    r = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                   case.q_seq, torch.tensor([-1], dtype=torch.int32))
    assert (r["sel"] == -1).all() and (r["out"] == 0).all()
    assert np.isneginf(r["scores"]).all()


# ----------------------------------------------------------------------------- page2d rotary
def _rand_vec(seed, n=128):
    return bf16(torch.randn(n, generator=torch.Generator().manual_seed(seed)))


def test_rope_constants_match_pages():
    g = json.load(open(GOLDEN))
    assert oracle.ROPE_PAGE_PAIRS == g["sparse_rope_page_pairs"]["value"]
    assert oracle.ROPE_PAGE_MOD == g["sparse_rope_page_mod"]["value"]
    assert oracle.ROPE_THETA_TOK == g["rope_theta_token_axis"]["value"]
    assert oracle.ROPE_THETA_PAGE == g["rope_theta_page_axis"]["value"]


def test_rope_identity_at_origin_and_even_pages():
    x = _rand_vec(1)
    for page in (0, 2, 10, -4):
        np.testing.assert_array_equal(oracle.rope_page2d(x, 0, page), x.double().numpy())


def test_rope_is_a_rotation_of_each_pair():
    x = _rand_vec(2).double().numpy()
    for tok, page in [(1, 0), (37, 1), (1000, 3), (131071, 0)]:
        y = oracle.rope_page2d(bf16(x), tok, page)
        np.testing.assert_allclose(y[:64] ** 2 + y[64:] ** 2, x[:64] ** 2 + x[64:] ** 2, rtol=1e-12, atol=1e-12)


def test_rope_dot_products_depend_only_on_the_token_offset():
    """Relative-position property: <R(t1) q, R(t2) k> is unchanged when both move by the same shift."""
    q, k = _rand_vec(3), _rand_vec(4)
    for page in (0, 1):
        base = oracle.rope_page2d(q, 5, page) @ oracle.rope_page2d(k, 12, page)
        for shift in (1, 17, 300, 40000):
            moved = oracle.rope_page2d(q, 5 + shift, page) @ oracle.rope_page2d(k, 12 + shift, page)
            assert abs(moved - base) < 1e-9


def test_rope_page_axis_is_page_parity():
    x = _rand_vec(5)
    for tok in (0, 9, 512):
        np.testing.assert_allclose(oracle.rope_page2d(x, tok, 1), oracle.rope_page2d(x, tok, 3), rtol=0, atol=0)
        np.testing.assert_allclose(oracle.rope_page2d(x, tok, 0), oracle.rope_page2d(x, tok, 8), rtol=0, atol=0)
    # same page parity, different token: differ; same token, other parity: differ only in the page pair
    a, b = oracle.rope_page2d(x, 9, 0), oracle.rope_page2d(x, 9, 1)
    diff = np.nonzero(np.abs(a - b) > 0)[0].tolist()
    assert diff and set(diff) <= {63, 127}


def test_rope_highest_frequencies():
    """Both axes start their spectrum at one radian per unit (theta ** 0): the token axis' first pair
    turns by `tok` radians, the page pair by (page % 2) radians."""
    e0 = torch.zeros(128)
    e0[0] = 1.0
    y = oracle.rope_page2d(bf16(e0), 1, 0)
    np.testing.assert_allclose([y[0], y[64]], [np.cos(1.0), np.sin(1.0)], rtol=0, atol=1e-15)
    e63 = torch.zeros(128)
    e63[63] = 1.0
    y = oracle.rope_page2d(bf16(e63), 12345, 1)
    np.testing.assert_allclose([y[63], y[127]], [np.cos(1.0), np.sin(1.0)], rtol=0, atol=1e-15)


def test_rope_token_spectrum_spans_theta():
    """'resample': 63 token frequencies spread over the whole spectrum from 1 down towards 1/theta.
    The angle of pair i after one step is recovered from the rotation of e_i and must fall
    monotonically from 1 to between 1/theta and its 63rd root above it."""
    angles = []
    for i in range(63):
        e = torch.zeros(128)
        e[i] = 1.0
        y = oracle.rope_page2d(bf16(e), 1, 0)
        angles.append(np.arctan2(y[i + 64], y[i]))
    angles = np.array(angles)
    assert angles[0] == pytest.approx(1.0, abs=1e-15)
    assert (np.diff(angles) < 0).all()
    assert 1e-4 < angles[-1] <= 1e-4 * 10000 ** (1 / 63) * (1 + 1e-12)
    ratios = angles[1:] / angles[:-1]
    np.testing.assert_allclose(ratios, ratios[0], rtol=1e-9)        # a geometric spectrum


def test_rope_append_writes_rotated_keys_and_raw_values():
    case = workloads.make_case([40, 70], heads=2, shuffle=True, seed=14)
    n, H = 2, 2
    g = torch.Generator().manual_seed(15)
    qn, kn, vn = (bf16(torch.randn(n, H, 128, generator=g)) for _ in range(3))
    qin, kin = (bf16(torch.randn(n, 128, generator=g)) for _ in range(2))
    tok, page, pos = np.array([3, 70]), np.array([0, 5]), np.array([39, 69])
    qr, qir, kc, vc, ic = oracle.rope_append(qn, qin, kn, vn, kin, tok, page, np.array([0, 1]), pos,
                                             case.block_table, case.k_pool, case.v_pool, case.idx_k_pool)
    for i in range(n):
        pg = int(case.block_table[i, pos[i] // 32])
        r = pos[i] % 32
        for h in range(H):
            np.testing.assert_array_equal(kc[pg, h, r], oracle.rope_page2d(kn[i, h], tok[i], page[i]))
            np.testing.assert_array_equal(vc[pg, h, r], vn[i, h].double().numpy())
            np.testing.assert_array_equal(qr[i, h], oracle.rope_page2d(qn[i, h], tok[i], page[i]))
        np.testing.assert_array_equal(ic[pg, r], oracle.rope_page2d(kin[i], tok[i], page[i]))
    # every other cache row is untouched
    untouched = np.ones(kc.shape[:3], bool)
    for i in range(n):
        untouched[int(case.block_table[i, pos[i] // 32]), :, pos[i] % 32] = False
    np.testing.assert_array_equal(kc[untouched], case.k_pool.double().numpy()[untouched])


# ----------------------------------------------------------------------------- summary scoring, masked selection
def test_summary_scores_brute_force():
    g = torch.Generator().manual_seed(21)
    qi = bf16(torch.randn(128, generator=g))
    summ = bf16(torch.randn(6, 128, generator=g))
    perm = np.array([3, 0, 5, 1, 4, 2])
    for p in [0, 31, 32, 100, 191]:
        s = oracle.summary_scores(qi, summ, perm, p)
        want = (summ.double()[perm[: p // 32 + 1]] @ qi.double()).numpy()
        np.testing.assert_allclose(s, want, rtol=0, atol=1e-12)


def test_mean_summary_score_is_the_mean_token_score():
    """Linearity: q . mean_t(k_t) = mean_t(q . k_t) -- ties the summary path to the per-token dots."""
    g = torch.Generator().manual_seed(22)
    qi = bf16(torch.randn(128, generator=g))
    pages = bf16(torch.randn(4, 32, 128, generator=g))
    for page in range(4):
        mean = oracle.block_mean(pages, page)
        dots = (pages[page].double() @ qi.double()).numpy()
        assert abs(mean @ qi.double().numpy() - dots.mean()) < 1e-10
        np.testing.assert_allclose(mean, pages[page].double().mean(0).numpy(), rtol=0, atol=1e-15)


def test_summary_of_a_constant_block_is_its_row():
    row = bf16(torch.linspace(-3, 3, 128))
    pages = row.expand(2, 32, 128).clone()
    np.testing.assert_array_equal(oracle.block_mean(pages, 1), row.double().numpy())


@pytest.mark.parametrize("seed", range(30))
def test_masked_select_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(0, 14))
    n_local, n_remote = int(rng.integers(0, 5)), int(rng.integers(0, 6))
    s = rng.integers(-3, 4, size=max(nb, 1)).astype(np.float64)
    allowed = rng.random(max(nb, 1)) < 0.6
    mask = np.zeros(1, np.uint32)
    for j in range(nb):
        if allowed[j]:
            mask[0] |= np.uint32(1 << j)
    sel, _ = oracle.select_masked(s, nb, mask, n_local, n_remote, tie_eps=0.5)
    cand = [j for j in range(max(nb - n_local, 0)) if allowed[j]]
    k = min(n_remote, len(cand))
    best, sets = None, []
    for comb in itertools.combinations(cand, k):
        tot = sum(s[j] for j in comb)
        if best is None or tot > best:
            best, sets = tot, [comb]
        elif tot == best:
            sets.append(comb)
    want = sorted(list(min(sets)) + list(range(max(nb - n_local, 0), nb)))
    assert sel.tolist() == want + [-1] * (n_local + n_remote - len(want))


def test_full_mask_equals_unmasked_selection():
    rng = np.random.default_rng(5)
    for nb in [0, 5, 16, 17, 40, 200]:
        s = rng.standard_normal(max(nb, 1))
        full = np.full((nb + 31) // 32 + 1, 0xFFFFFFFF, np.uint32)
        a, ta = oracle.select(s, nb)
        b, tb = oracle.select_masked(s, nb, full)
        assert np.array_equal(a, b) and ta == tb
