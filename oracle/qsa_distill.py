"""Plain fp64 CPU oracle of the indexer's distillation signal -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module; the product path never calls it and shares no code with it.  Inputs are numpy arrays
of bf16 bit patterns, computed in float64, step by step.

Source: the article "Qwen's million-token window has a 2,048-token keyhole" (cronfeed.work),
section "The indexer is trained, not bolted on" (Chinese edition: "索引器靠训练融入模型").  Before
sparse training, the indexer was warmed up by dense distillation: it learned from the full
(dense) attention distribution while the rest of the model stayed frozen, and the teacher signal
was token-level attention pooled into blocks.

The article gives no formula.  The readings taken here, the plainest the text supports:
  * teacher: for query position t, the dense causal softmax attention of every core query head
    over positions 0..t (softmax scale 1/sqrt(D), query head h reading key head h // (Hq/Hkv)),
    pooled into 4-token micro-blocks by summing each block's probabilities, summed over all query
    heads, restricted to the indexer's candidate blocks b < t // 4 and renormalised to sum 1.  The
    block holding t is left out: it is always selected and never ranked;
  * student: the softmax, over the same candidate blocks, of the indexer's block scores
    s_b = sum_h w_h * max(0, q_h . k_b) (the selection scores, temperature 1);
  * loss: KL(teacher || student) per query row, in nats; a row with no candidate (t < 4) has
    loss 0.

Pins (tests/test_oracle_distill.py): the block pooling against torch's fp64 attention with
one-hot block indicators as values, the uniform-attention closed form, a dominant-position case,
scipy's softmax and relative entropy, and the KL against a uniform student.  No function here
is unpinned.
"""
from __future__ import annotations

import math

import numpy as np

from .qsa_oracle import BLOCK_TOKENS, bf16_to_f64, block_scores, num_candidates


def dense_attention_probs(q_bits: np.ndarray, k_bits: np.ndarray, t: int,
                          scale: float | None = None) -> np.ndarray:
    """Dense causal attention probabilities of one query at position t.

    q_bits: bf16 [Hq, D]; k_bits: bf16 [>= t+1, Hkv, D] keys of positions 0.. of its sequence.
    Returns a [Hq, t+1]: row h is the softmax over positions 0..t of scale * q_h . k_p, with key
    head h // (Hq // Hkv)."""
    q = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_bits[: t + 1])
    hq, d = q.shape
    group = hq // k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    a = np.zeros((hq, t + 1), dtype=np.float64)
    for h in range(hq):
        z = (k[:, h // group, :] @ q[h]) * scale
        e = np.exp(z - z.max())
        a[h] = e / e.sum()
    return a


def teacher_blocks(probs: np.ndarray, t: int, block: int = BLOCK_TOKENS) -> np.ndarray:
    """The distillation target of one query at position t: the attention probabilities probs
    [Hq, t+1] summed over the tokens of each candidate block b < t // block and over the heads,
    then divided by their total.  Returns [t // block] (empty when there is no candidate)."""
    n = num_candidates(t, block)
    if n == 0:
        return np.zeros(0, dtype=np.float64)
    mass = probs[:, : n * block].sum(axis=0).reshape(n, block).sum(axis=1)
    return mass / mass.sum()


def indexer_softmax(scores: np.ndarray) -> np.ndarray:
    """The indexer's distribution over candidate blocks: softmax of its block scores."""
    if scores.size == 0:
        return np.zeros(0, dtype=np.float64)
    e = np.exp(scores - scores.max())
    return e / e.sum()


def kl_divergence(p: np.ndarray, q: np.ndarray) -> float:
    """KL(p || q) = sum_b p_b log(p_b / q_b) in nats; terms with p_b = 0 contribute 0."""
    nz = p > 0
    return float(np.sum(p[nz] * (np.log(p[nz]) - np.log(q[nz]))))


def distill_row(kcomp_bits, idx_q_bits, idx_w_bits, q_bits, k_seq_bits, t: int,
                block: int = BLOCK_TOKENS, scale: float | None = None):
    """Distillation loss of one query at position t.  Returns (kl, teacher [t//4], student
    [t//4], lse [Hq]) where lse is the natural-log normaliser of each head's dense softmax."""
    n = num_candidates(t, block)
    probs = dense_attention_probs(q_bits, k_seq_bits, t, scale)
    p = teacher_blocks(probs, t, block)
    s = block_scores(kcomp_bits, idx_q_bits, idx_w_bits, n)
    q = indexer_softmax(s)
    qf = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_seq_bits[: t + 1])
    group = qf.shape[0] // k.shape[1]
    sc = 1.0 / math.sqrt(qf.shape[1]) if scale is None else scale
    lse = np.zeros(qf.shape[0], dtype=np.float64)
    for h in range(qf.shape[0]):
        z = (k[:, h // group, :] @ qf[h]) * sc
        m = z.max()
        lse[h] = m + math.log(np.exp(z - m).sum())
    kl = kl_divergence(p, q) if n else 0.0
    return kl, p, q, lse
