"""Seeded synthetic inputs shared by the CUDA path's tests / bench and the oracle.

This module holds no arithmetic of the attention method: it only draws the
tensors a decode or prefill step consumes (queries, paged K/V caches, the
indexer key cache, block tables, lengths) with the shapes and value
distributions of the Unlimited-OCR-2 workloads:

* 10 heads x 128 dims MHA and a 1-head x 128-dim indexer
  (Unlimited-OCR-2 walk-through, news.rkmt.cn/news/25027, section 三);
* 32-token KV blocks (same page, section 五 step 1);
* contexts up to 131072 tokens (same page, section 三: YaRN to 128K).

Recipe (stated once, used everywhere):
  1. Structural integers come from a CPU ``torch.Generator`` seeded with
     ``seed``, in this order: ragged lengths, physical page permutation,
     planted blocks and offsets.  They are identical on every device.
  2. Values come from a ``torch.Generator`` on ``device`` seeded with ``seed``,
     in this order: q, idx_q, then per layer k_pool, v_pool, idx_k_pool.  Each is
     N(0,1) drawn in fp32 in chunks of at most ``_CHUNK`` elements and rounded
     to bf16 (round-to-nearest-even by ``Tensor.to``).
  3. Planted references: ``idx_k[t] <- bf16(float(idx_k[t]) + 0.5*float(idx_q))``
     at 3 distinct offsets of each planted block.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLOCK = 32
HEADS = 10
HEAD_DIM = 128
IDX_DIM = 128
_CHUNK = 1 << 26


@dataclass
class Case:
    """One batch of decode/prefill input.  ``layers`` holds per-layer cache triples."""
    q: torch.Tensor              # [n_q, H, D] bf16 (layer 0; per-layer copies in q_layers)
    idx_q: torch.Tensor          # [n_q, IDX_DIM] bf16
    block_table: torch.Tensor    # [B, max_blocks] int32 (-1 past a sequence's blocks)
    seq_lens: torch.Tensor       # [B] int32
    q_seq: torch.Tensor          # [n_q] int32
    q_pos: torch.Tensor          # [n_q] int32
    layers: list = field(default_factory=list)   # [(k_pool, v_pool, idx_k_pool)] per layer
    q_layers: list = field(default_factory=list)      # [(q, idx_q)] per layer
    planted: dict = field(default_factory=dict)       # seq -> list of planted logical blocks
    num_pages: int = 0
    name: str = ""

    @property
    def k_pool(self):
        return self.layers[0][0]

    @property
    def v_pool(self):
        return self.layers[0][1]

    @property
    def idx_k_pool(self):
        return self.layers[0][2]

    @property
    def n_q(self):
        return int(self.q_seq.shape[0])

    @property
    def max_blocks(self):
        return int(self.block_table.shape[1])


def randn_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) in fp32, rounded to bf16, drawn in bounded chunks along a flat view."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def make_case(seq_lens, *, n_layers: int = 1, heads: int = HEADS, shuffle: bool = False,
              planted_blocks: int = 0, planted_tokens: int = 3, max_blocks: int | None = None,
              q_pos: list | None = None, q_seq: list | None = None, seed: int = 0,
              device="cpu", name: str = "") -> Case:
    """Draw one case.

    seq_lens        tokens cached per sequence (the decode query is the last of them).
    shuffle         scatter the pages over the pool in a random physical order.
    planted_blocks  per sequence, this many distinct remote-candidate blocks get
                    ``planted_tokens`` distinct offsets with +0.5*idx_q added.
    q_pos / q_seq   explicit query positions (prefill); default one decode query
                    per sequence at p = seq_len - 1.
    """
    device = torch.device(device)
    seq_lens = [int(x) for x in seq_lens]
    B = len(seq_lens)
    nbs = [(L + BLOCK - 1) // BLOCK for L in seq_lens]
    mb = max_blocks if max_blocks is not None else max(max(nbs), 1)
    assert mb >= max(nbs)
    P = sum(nbs)

    g_cpu = torch.Generator().manual_seed(seed)
    perm = torch.randperm(P, generator=g_cpu) if shuffle else torch.arange(P)
    bt = torch.full((B, mb), -1, dtype=torch.int32)
    off = 0
    for b, nb in enumerate(nbs):
        bt[b, :nb] = perm[off:off + nb].to(torch.int32)
        off += nb

    if q_seq is None:
        q_seq = list(range(B))
        q_pos = [L - 1 for L in seq_lens]
    n_q = len(q_seq)

    planted = {}
    if planted_blocks:
        for b, nb in enumerate(nbs):
            n_cand = nb - 4
            assert n_cand >= planted_blocks, "not enough remote candidates to plant"
            blocks = torch.randperm(n_cand, generator=g_cpu)[:planted_blocks].tolist()
            offs = [torch.randperm(BLOCK, generator=g_cpu)[:planted_tokens].tolist() for _ in blocks]
            planted[b] = list(zip(blocks, offs))

    g = torch.Generator(device=device).manual_seed(seed)
    case = Case(q=None, idx_q=None, block_table=bt.to(device), seq_lens=torch.tensor(seq_lens, dtype=torch.int32, device=device),
                q_seq=torch.tensor(q_seq, dtype=torch.int32, device=device),
                q_pos=torch.tensor(q_pos, dtype=torch.int32, device=device), num_pages=P, name=name)
    for layer in range(n_layers):
        q = randn_bf16((n_q, heads, HEAD_DIM), g, device)
        qi = randn_bf16((n_q, IDX_DIM), g, device)
        case.q_layers.append((q, qi))
    for layer in range(n_layers):
        kp = randn_bf16((P, heads, BLOCK, HEAD_DIM), g, device)
        vp = randn_bf16((P, heads, BLOCK, HEAD_DIM), g, device)
        ikp = randn_bf16((P, BLOCK, IDX_DIM), g, device)
        if planted:
            qi = case.q_layers[layer][1]
            for b, items in planted.items():
                # the query of sequence b (decode: one query per sequence)
                qrow = q_seq.index(b)
                for j, offs in items:
                    page = int(bt[b, j])
                    for o in offs:
                        ikp[page, o] = (ikp[page, o].float() + 0.5 * qi[qrow].float()).to(torch.bfloat16)
        case.layers.append((kp, vp, ikp))
    case.q, case.idx_q = case.q_layers[0]
    case.planted = {b: [j for j, _ in items] for b, items in planted.items()}
    return case


# --------------------------------------------------------------------------- named workloads
def ragged_lengths(B: int, lo_blocks: int, hi_blocks: int, seed: int) -> list:
    """Context lengths 32*randint(lo, hi) inclusive: uniform, rounded to whole 32-token blocks."""
    g = torch.Generator().manual_seed(seed)
    return [BLOCK * int(x) for x in torch.randint(lo_blocks, hi_blocks + 1, (B,), generator=g)]


def tiny_decode(device="cpu", seed=0) -> Case:
    """Batch 1, context 2048 (64 blocks), one decode query."""
    return make_case([2048], seed=seed, device=device, name="tiny_decode_b1_ctx2048")


def batched_decode(device="cpu", seed=0, B=16, L=32768) -> Case:
    """Batch 16, context 32768 (1024 blocks), 12 planted reference blocks per sequence."""
    return make_case([L] * B, planted_blocks=12, seed=seed, device=device,
                     name=f"batched_decode_b{B}_ctx{L}_planted12")


def long_decode(device="cpu", seed=0, B=16, L=131072, n_layers=12) -> Case:
    """Batch 16, context 131072 (4096 blocks), 12 independent layer caches."""
    return make_case([L] * B, n_layers=n_layers, seed=seed, device=device,
                     name=f"long_decode_b{B}_ctx{L}_layers{n_layers}")


def ragged_paged_decode(device="cpu", seed=0, B=64, lo_blocks=128, hi_blocks=4096, max_blocks=4096) -> Case:
    """Batch 64, lengths uniform in [4096, 131072] rounded to 32, pages shuffled in one pool."""
    lens = ragged_lengths(B, lo_blocks, hi_blocks, seed)
    return make_case(lens, shuffle=True, max_blocks=max_blocks, seed=seed, device=device,
                     name=f"ragged_paged_decode_b{B}_ctx{lo_blocks * BLOCK}-{hi_blocks * BLOCK}")


def chunked_prefill(device="cpu", seed=0, prefix=63488, n_new=2048) -> Case:
    """One sequence, n_new causal queries appended to a prefix (their K/V already cached)."""
    total = prefix + n_new
    return make_case([total], q_seq=[0] * n_new, q_pos=list(range(prefix, total)), seed=seed,
                     device=device, name=f"chunked_prefill_{n_new}q_ctx{total}")
