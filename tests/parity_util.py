"""Comparison of the CUDA path with the fp64 oracle, query by query.

For each checked query the oracle gets only what it needs, read back from the
device: the sequence's indexer pages (for scores and selection) and the K/V
pages of the selected blocks (for attention), re-indexed into small host
pools.  That lets full-size workloads be checked on sampled queries.

``check_all_queries`` does the same for every query of a one-sequence case
(a prefill chunk) with one host copy of the sequence's pages and the oracle
run over all queries at once (OpenMP).

Acceptance (per query):
  * block scores: |gpu - oracle| <= SCORE_ATOL on every causal block;
  * selection: identical to the oracle's, unless the oracle flags a near tie
    (12th and 13th remote scores closer than 1e-3); then the GPU set G is
    accepted iff it holds every candidate scoring above s_(13) + 1e-3 and
    nothing scoring below s_(12) - 1e-3, and the output is compared with the
    oracle's attention over G;
  * output: max |gpu - oracle| <= OUT_MAX_ATOL and mean <= OUT_MEAN_ATOL.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

SCORE_ATOL = 1e-3
OUT_MAX_ATOL = 2e-2
OUT_MEAN_ATOL = 2e-3
TIE = 1e-3


def _query_inputs(case, layer, i):
    b = int(case.q_seq[i])
    p = int(case.q_pos[i])
    nb = p // 32 + 1 if p >= 0 else 0
    return b, p, nb


def oracle_scores_and_sel(case, i, layer=0):
    """fp64 scores [nb] and (sel, near_tie) for query i, from the sequence's indexer pages only."""
    _, idx_q = case.q_layers[layer]
    ikp = case.layers[layer][2]
    b, p, nb = _query_inputs(case, layer, i)
    if nb == 0:
        return np.zeros(0), np.full(16, -1, np.int32), False
    pages = case.block_table[b, :nb].long()
    mini = ikp[pages].cpu()
    s = oracle.block_scores(idx_q[i].cpu(), mini, np.arange(nb), p)
    sel, tie = oracle.select(s, nb)
    return s, sel, tie


def oracle_attend(case, i, sel, layer=0, scale=None):
    q, _ = case.q_layers[layer]
    kp, vp, _ = case.layers[layer]
    b, p, nb = _query_inputs(case, layer, i)
    sel = np.asarray(sel, np.int32)
    used = [int(j) for j in sel if j >= 0]
    H = q.shape[1]
    if not used:
        return np.zeros((H, 128))
    pages = case.block_table[b, torch.tensor(used, dtype=torch.long)].long()
    mk, mv = kp[pages].cpu(), vp[pages].cpu()
    bt = np.full(max(nb, 1), -1, np.int32)
    for n, j in enumerate(used):
        bt[j] = n
    return oracle.attend(q[i].cpu(), mk, mv, bt, sel, p, scale=scale)


def accept_selection(s, sel_oracle, sel_gpu, tie):
    """True if the GPU selection is the oracle's, or an admissible answer to a near tie."""
    if np.array_equal(sel_oracle, sel_gpu):
        return True
    if not tie:
        return False
    nb = s.shape[0]
    cand = s[: nb - 4]
    order = np.sort(cand)[::-1]
    s12, s13 = order[11], order[12]
    g = [int(j) for j in sel_gpu if j >= 0]
    if sorted(g) != list(sel_gpu[: len(g)]) or len(g) != 16:
        return False
    if g[12:] != list(range(nb - 4, nb)):
        return False
    remote = set(g[:12])
    must = {j for j in range(nb - 4) if cand[j] > s13 + TIE}
    return must <= remote and all(cand[j] >= s12 - TIE for j in remote)


def check_queries(case, queries, out_gpu, sel_gpu, scores_gpu=None, layer=0, report=None):
    """Assert parity for the listed queries; returns per-query error stats."""
    out_gpu = out_gpu.float().cpu().numpy()
    sel_gpu = sel_gpu.cpu().numpy()
    sc = scores_gpu.cpu().numpy() if scores_gpu is not None else None
    stats = []
    for i in queries:
        s, sel_o, tie = oracle_scores_and_sel(case, i, layer)
        nb = s.shape[0]
        if sc is not None and nb:
            err = np.abs(sc[i, :nb].astype(np.float64) - s).max()
            assert err <= SCORE_ATOL, f"query {i}: score error {err}"
        assert accept_selection(s, sel_o, sel_gpu[i], tie), \
            f"query {i}: selection {sel_gpu[i].tolist()} vs oracle {sel_o.tolist()} (near tie {tie})"
        ref = oracle_attend(case, i, sel_gpu[i], layer)
        d = np.abs(out_gpu[i] - ref)
        assert d.max() <= OUT_MAX_ATOL and d.mean() <= OUT_MEAN_ATOL, \
            f"query {i}: out max {d.max()} mean {d.mean()}"
        stats.append((i, float(d.max()), float(d.mean()), bool(tie)))
    if report is not None:
        report.extend(stats)
    return stats


def check_all_queries(case, out_gpu, sel_gpu, scores_gpu=None, layer=0, threads=0):
    """check_queries for every query of a case whose queries all belong to one sequence, with the
    sequence's pages copied to the host once and the oracle run over all queries in one call.
    Returns (max abs error, mean abs error, near ties) over all queries."""
    q, idx_q = case.q_layers[layer]
    kp, vp, ikp = case.layers[layer]
    seqs = set(case.q_seq.cpu().tolist())
    assert len(seqs) == 1, "one sequence only"
    b = seqs.pop()
    nb_max = int(case.q_pos.max().item()) // 32 + 1
    pages = case.block_table[b, :nb_max].long()
    h_idx, h_k, h_v = ikp[pages].cpu(), kp[pages].cpu(), vp[pages].cpu()
    bt = np.arange(nb_max, dtype=np.int32).reshape(1, nb_max)     # logical block j -> host page j
    qs = np.zeros(case.n_q, np.int32)
    qp = case.q_pos.cpu().numpy().astype(np.int32)
    h_q, h_qi = q.cpu(), idx_q.cpu()
    r = oracle.run(h_q, h_qi, h_k[:1], h_v[:1], h_idx, bt, qs, qp, want_out=False, threads=threads)
    sel = sel_gpu.cpu().numpy()
    sc = scores_gpu.cpu().numpy() if scores_gpu is not None else None
    ties = 0
    for i in range(case.n_q):
        nb = int(qp[i]) // 32 + 1 if qp[i] >= 0 else 0
        s = r["scores"][i, :nb]
        if sc is not None and nb:
            err = np.abs(sc[i, :nb].astype(np.float64) - s).max()
            assert err <= SCORE_ATOL, f"query {i}: score error {err}"
        tie = bool(r["near_tie"][i])
        ties += int(tie)
        assert accept_selection(s, r["sel"][i], sel[i], tie), \
            f"query {i}: selection {sel[i].tolist()} vs oracle {r['sel'][i].tolist()} (near tie {tie})"
    ref = oracle.run(h_q, h_qi, h_k, h_v, h_idx[:1], bt, qs, qp, sel_in=sel, threads=threads)["out"]
    got = out_gpu.float().cpu().numpy()
    d = np.abs(got - ref)
    per_max = d.reshape(case.n_q, -1).max(axis=1)
    per_mean = d.reshape(case.n_q, -1).mean(axis=1)
    bad = np.nonzero((per_max > OUT_MAX_ATOL) | (per_mean > OUT_MEAN_ATOL))[0]
    assert bad.size == 0, f"queries {bad[:10].tolist()}: out max {per_max[bad[:10]].tolist()}"
    return float(d.max()), float(d.mean()), ties
