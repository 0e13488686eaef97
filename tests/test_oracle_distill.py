"""Pins of the distillation oracle (oracle/qsa_distill.py) against things other than itself.

The method text is the article "Qwen's million-token window has a 2,048-token keyhole", section
"The indexer is trained, not bolted on": the indexer was first distilled from the full-attention
distribution, with token-level attention pooled into blocks as the teacher.  Each pin ties one
step to an independent route (torch's fp64 attention, scipy's softmax and relative entropy) or a
closed form.
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

from oracle import qsa_distill as dst
from oracle import qsa_oracle as orc


def rand_bits(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f64(bits):
    return orc.bf16_to_f64(bits)


@pytest.mark.parametrize("hq,hkv,d,t", [(4, 1, 64, 37), (8, 2, 32, 64), (6, 3, 16, 5)])
def test_teacher_pooling_matches_attention_with_block_indicator_values(hq, hkv, d, t):
    """Pooling through another route: torch's fp64 attention whose values are one-hot block
    indicators returns, per head, the attention mass of each block; summed over heads, the
    candidate entries renormalised must equal the oracle's teacher."""
    rng = np.random.default_rng(10 + t)
    q = rand_bits(rng, (hq, d))
    k = rand_bits(rng, (t + 1, hkv, d))
    nb = t // 4 + 1
    onehot = np.zeros((t + 1, nb))
    onehot[np.arange(t + 1), np.arange(t + 1) // 4] = 1.0
    qt = torch.tensor(f64(q))[None, :, None, :]                                   # [1, Hq, 1, D]
    kt = torch.tensor(f64(k)).repeat_interleave(hq // hkv, dim=1).permute(1, 0, 2)[None]
    vt = torch.tensor(onehot)[None, None].expand(1, hq, t + 1, nb)
    mass = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0, :].sum(0).numpy()
    want = mass[: t // 4] / mass[: t // 4].sum()
    got = dst.teacher_blocks(dst.dense_attention_probs(q, k, t), t)
    assert got.shape == (t // 4,)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
    assert abs(got.sum() - 1.0) < 1e-12


def test_dense_probs_are_a_softmax_matching_torch():
    rng = np.random.default_rng(11)
    q, k, t = rand_bits(rng, (4, 32)), rand_bits(rng, (50, 2, 32)), 41
    a = dst.dense_attention_probs(q, k, t)
    logits = torch.tensor(f64(q)) @ torch.tensor(f64(k[: t + 1])).repeat_interleave(2, dim=1).permute(1, 2, 0)
    ref = torch.softmax(torch.diagonal(logits, dim1=0, dim2=1).T / math.sqrt(32), dim=-1).numpy()
    assert np.allclose(a, ref, rtol=1e-12, atol=1e-15)


def test_uniform_attention_gives_uniform_teacher():
    """q = 0: every position gets 1/(t+1); every candidate block holds 4 of them, so the
    renormalised teacher is exactly uniform over the t // 4 candidates."""
    rng = np.random.default_rng(12)
    t = 103
    q = np.zeros((4, 16), dtype=np.uint16)   # bf16 +0
    k = rand_bits(rng, (t + 1, 1, 16))
    p = dst.teacher_blocks(dst.dense_attention_probs(q, k, t), t)
    assert p.shape == (25,)
    assert np.allclose(p, 1.0 / 25, rtol=1e-14, atol=0)


def test_dominant_position_pools_to_its_block():
    """One key aligned with every head's query and far larger than the rest: nearly all of the
    attention mass sits at that position, so the teacher is nearly one-hot on its block."""
    rng = np.random.default_rng(13)
    t, d, star = 60, 16, 22
    q = np.zeros((4, d), dtype=np.float32)
    q[:, 0] = 1.0
    k = rng.uniform(-0.1, 0.1, (t + 1, 1, d)).astype(np.float32)
    k[star, 0, 0] = 64.0                      # logit 16 above the rest after the 1/sqrt(16) scale
    qb = torch.tensor(q).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kb = torch.tensor(k).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    p = dst.teacher_blocks(dst.dense_attention_probs(qb, kb, t), t)
    assert np.argmax(p) == star // 4 and p[star // 4] > 0.9999


def test_tail_block_is_excluded_and_short_rows_are_empty():
    rng = np.random.default_rng(14)
    k = rand_bits(rng, (12, 1, 8))
    q = rand_bits(rng, (2, 8))
    for t in range(4):
        assert dst.teacher_blocks(dst.dense_attention_probs(q, k, t), t).size == 0
    a = dst.dense_attention_probs(q, k, 9)       # candidates: blocks 0, 1; block 2 holds t = 9
    p = dst.teacher_blocks(a, 9)
    m = a.sum(0)
    assert np.allclose(p, [m[0:4].sum() / m[0:8].sum(), m[4:8].sum() / m[0:8].sum()], rtol=1e-13)


def test_student_softmax_and_kl_match_scipy():
    rng = np.random.default_rng(15)
    s = rng.standard_normal(300) * 7
    q = dst.indexer_softmax(s)
    assert np.allclose(q, scipy.special.softmax(s), rtol=1e-13, atol=0)
    p = rng.dirichlet(np.ones(300))
    p[::7] = 0.0
    p /= p.sum()
    assert math.isclose(dst.kl_divergence(p, q), scipy.stats.entropy(p, q), rel_tol=1e-12)
    assert dst.kl_divergence(p, p) == 0.0
    assert dst.kl_divergence(p, q) > 0


def test_distill_row_with_zero_weights_is_kl_to_uniform():
    """Zero head weights make every block score 0, so the student is uniform and the loss is
    log(n) minus the teacher's entropy; the lse output matches torch's logsumexp."""
    rng = np.random.default_rng(16)
    t, hq, hkv, d, di = 77, 4, 2, 32, 16
    kc = rand_bits(rng, (t // 4 + 1, di))
    iq = rand_bits(rng, (4, di))
    iw = np.zeros(4, dtype=np.uint16)
    q = rand_bits(rng, (hq, d))
    k = rand_bits(rng, (t + 1, hkv, d))
    kl, p, s, lse = dst.distill_row(kc, iq, iw, q, k, t)
    n = t // 4
    assert np.allclose(s, 1.0 / n, rtol=1e-14, atol=0)
    assert math.isclose(kl, math.log(n) - scipy.stats.entropy(p), rel_tol=1e-10)
    logits = (torch.tensor(f64(k)).repeat_interleave(2, dim=1).permute(1, 0, 2) @
              torch.tensor(f64(q))[:, :, None])[:, :, 0] / math.sqrt(d)
    assert np.allclose(lse, torch.logsumexp(logits, dim=1).numpy(), rtol=1e-13)


def test_distill_row_student_uses_the_selection_scores():
    """The student's logits are the indexer's block scores: a row whose teacher equals the
    softmax of those scores would have loss 0, and the loss against the real teacher is the
    relative entropy scipy computes from the same two distributions."""
    rng = np.random.default_rng(17)
    t, di = 201, 32
    kc = rand_bits(rng, (t // 4 + 1, di))
    iq = rand_bits(rng, (4, di))
    iw = rand_bits(rng, 4)
    q = rand_bits(rng, (4, 16))
    k = rand_bits(rng, (t + 1, 1, 16))
    kl, p, s, _ = dst.distill_row(kc, iq, iw, q, k, t)
    sc = orc.block_scores(kc, iq, iw, t // 4)
    assert np.allclose(s, scipy.special.softmax(sc), rtol=1e-13)
    assert math.isclose(kl, scipy.stats.entropy(p, scipy.special.softmax(sc)), rel_tol=1e-12)
