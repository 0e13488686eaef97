"""Plain fp64 CPU oracle of the QSA layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module.  The product path (the CUDA library and its Python binding) never calls it, and it
shares no code with that path: it takes plain numpy arrays of bf16 bit patterns and computes in
float64, step by step, in the order the method is described.

Source: the article "Qwen's million-token window has a 2,048-token keyhole" (cronfeed.work),
section "A million-token window with a selective view" (the Chinese edition of the same article
says the same in section "百万 token 窗口里的选择性视野").  In each QSA layer an indexer (four query
heads against a single key head) averages its keys over groups of four tokens, ranks those
groups, retains at most 512 of them -- a 2,048-token budget that does not grow with the context --
together with the still-open group at the end of the sequence (the article's opening
paragraphs), maps the retained groups back to their token positions, and runs the core attention
on those positions alone.  The comparison baseline is paged
grouped-query attention (section "Three speed claims, three different experiments").

The article leaves these steps open; the oracle takes the plainest reading, stated per function:
  * compression operator: the mean of the 4 raw indexer keys of a block, stored as bf16
    (round to nearest even of the exact fp64 mean);
  * block score: s_b = sum_h w_h * max(0, q_h . k_b), heads h = 0..3, per-query head weights w_h;
  * eligibility: block b is a candidate for query position t iff 4b + 3 <= t and b is not the
    block containing t, i.e. b < t // 4; the block containing t (the "tail") is always kept and
    does not count against the budget;
  * ranking: score descending, ties to the lower block index;
  * one selection per query token, shared by every core-attention head;
  * GQA mapping: query head h reads key/value head h // (Hq / Hkv); softmax scale 1/sqrt(D).

Parity pins live in tests/test_oracle.py (hand-worked golden fixture, closed forms, brute force,
and torch's scaled_dot_product_attention in fp64 as the textbook attention).  No function here
is unpinned.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK_TOKENS = 4     # tokens per micro-block of the compressed indexer key
TOPK_BLOCKS = 512    # micro-block budget per query (2,048 tokens)


# ----------------------------------------------------------------------------- bf16 helpers

def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits), nearest-even, return bit patterns.

    Written from the definition: x = m * 2**e with 0.5 <= |m| < 1; keep 8 significant bits by
    rounding m * 2**8 to the nearest integer, ties to even (np.rint); the result is exact in fp32,
    whose top 16 bits are the bf16 pattern.  Values here are far from bf16's exponent limits.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    r = np.rint(m * 256.0)
    y = np.ldexp(r, e - 8)
    return (y.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------- the steps

def compress(kidx_bits: np.ndarray, block: int = BLOCK_TOKENS) -> np.ndarray:
    """Micro-block compression of the shared indexer key head.

    kidx_bits: bf16 [n, Di] raw indexer keys of consecutive positions 0..n-1.
    Returns bf16 [n // block, Di]: k_b = bf16(mean of rows block*b .. block*b + block - 1).
    Only complete blocks are produced.
    """
    k = bf16_to_f64(kidx_bits)
    nb = k.shape[0] // block
    sums = np.zeros((nb, k.shape[1]), dtype=np.float64)
    for i in range(block):
        sums += k[i:nb * block:block]
    return f64_to_bf16_bits(sums / block)


def num_candidates(t: int, block: int = BLOCK_TOKENS) -> int:
    """Number of candidate blocks for query position t: blocks b < t // block (complete, and not
    the block holding t)."""
    return t // block


def block_scores(kcomp_bits: np.ndarray, idx_q_bits: np.ndarray, idx_w_bits: np.ndarray,
                 n_cand: int) -> np.ndarray:
    """Indexer score of candidate blocks 0..n_cand-1 for one query token, in fp64.

    kcomp_bits: bf16 [>= n_cand, Di]; idx_q_bits: bf16 [Hi, Di]; idx_w_bits: bf16 [Hi].
    s_b = sum over heads h (in order) of w_h * max(0, q_h . k_b).
    """
    kc = bf16_to_f64(kcomp_bits[:n_cand])
    q = bf16_to_f64(idx_q_bits)
    w = bf16_to_f64(idx_w_bits)
    s = np.zeros(n_cand, dtype=np.float64)
    for h in range(q.shape[0]):
        s += w[h] * np.maximum(kc @ q[h], 0.0)
    return s


def select_blocks(scores: np.ndarray, t: int, topk: int = TOPK_BLOCKS,
                  block: int = BLOCK_TOKENS) -> np.ndarray:
    """Top-``topk`` candidate blocks by (score descending, block ascending), plus the tail block
    t // block; returned in ascending block order (the tail, being the largest, is last)."""
    n = num_candidates(t, block)
    assert scores.shape[0] == n
    blocks = np.arange(n, dtype=np.int64)
    order = np.lexsort((blocks, -scores))          # primary: -score, secondary: block
    kept = np.sort(blocks[order[:min(topk, n)]])
    return np.concatenate([kept, np.array([t // block], dtype=np.int64)])


def expand(sel: np.ndarray, t: int, block: int = BLOCK_TOKENS) -> np.ndarray:
    """Token positions of the selected blocks that are causally visible (<= t), ascending."""
    pos = (np.asarray(sel, dtype=np.int64)[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    return pos[pos <= t]


def attend(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
           scale: float | None = None):
    """Softmax attention of one query token over the given key/value rows, fp64.

    q_bits: bf16 [Hq, D]; k_bits, v_bits: bf16 [P, Hkv, D] (rows in ascending position order).
    Query head h reads key/value head h // (Hq // Hkv).  Returns (o [Hq, D], lse [Hq]) with
    lse = natural log of the softmax normaliser of the scaled logits.
    """
    q = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_bits)
    v = bf16_to_f64(v_bits)
    hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.zeros((hq, d), dtype=np.float64)
    lse = np.zeros(hq, dtype=np.float64)
    for h in range(hq):
        g = h // group
        z = (k[:, g, :] @ q[h]) * scale
        m = z.max()
        e = np.exp(z - m)
        denom = e.sum()
        o[h] = (e @ v[:, g, :]) / denom
        lse[h] = m + math.log(denom)
    return o, lse


def dense_causal(q_bits: np.ndarray, k_all_bits: np.ndarray, v_all_bits: np.ndarray, t: int,
                 scale: float | None = None):
    """Dense causal grouped-query attention of one query at position t over positions 0..t
    (the paged-GQA baseline).  Written separately from ``attend``: the key/value heads are
    broadcast to query heads first and the softmax runs on a masked logit matrix."""
    q = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_all_bits)
    v = bf16_to_f64(v_all_bits)
    hq, d = q.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    kx = np.repeat(k, hq // hkv, axis=1)               # [P, Hq, D]
    vx = np.repeat(v, hq // hkv, axis=1)
    logits = np.einsum("hd,phd->hp", q, kx) * scale    # [Hq, P]
    mask = np.arange(k.shape[0]) <= t
    logits = np.where(mask[None, :], logits, -np.inf)
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    z = p.sum(axis=1, keepdims=True)
    o = np.einsum("hp,phd->hd", p / z, vx)
    return o, (mx + np.log(z))[:, 0]


# ----------------------------------------------------------------------------- one query row

def qsa_select(kcomp_bits: np.ndarray, idx_q_bits: np.ndarray, idx_w_bits: np.ndarray, t: int,
               topk: int = TOPK_BLOCKS, block: int = BLOCK_TOKENS):
    """Indexer path for one query at position t: scores of all candidates and the selection.
    Returns (sel ascending incl. tail, scores of all candidates)."""
    n = num_candidates(t, block)
    s = block_scores(kcomp_bits, idx_q_bits, idx_w_bits, n)
    return select_blocks(s, t, topk, block), s


def qsa_row(kcomp_bits, idx_q_bits, idx_w_bits, q_bits, k_seq_bits, v_seq_bits, t: int,
            topk: int = TOPK_BLOCKS, block: int = BLOCK_TOKENS, scale: float | None = None):
    """Whole QSA layer for one query at position t of a sequence whose K/V rows (position
    order, [>= t+1, Hkv, D]) are given.  Returns (o, lse, sel)."""
    sel, _ = qsa_select(kcomp_bits, idx_q_bits, idx_w_bits, t, topk, block)
    pos = expand(sel, t, block)
    o, lse = attend(q_bits, k_seq_bits[pos], v_seq_bits[pos], scale)
    return o, lse, sel
